"""The C-ABI library loads on a machine without a GPU, exports every symbol the
header declares, and rejects bad arguments on the host before touching a GPU."""
import ctypes
import os
import re

import pytest

from learnable_channel_permutation_b200 import binding as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lcp.h")

pytestmark = pytest.mark.skipif(not os.path.exists(b.LIB_PATH), reason="liblcp.so not built")


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^LCP_API\s+[\w\s\*]+?\b(\w+)\s*\(", txt, flags=re.M)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for name in ["lcp_sinkhorn_fwd", "lcp_sinkhorn_bwd", "lcp_permute_weight", "nm_mask", "lcp_loss_fwd",
                 "lcp_loss_bwd", "lcp_step", "lcp_workspace_size", "lcp_status_string"]:
        assert name in syms


def test_library_exports_every_declared_symbol():
    L = b.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert L.lcp_abi_version() == int(re.search(r"#define LCP_ABI_VERSION (\d+)", open(HEADER).read()).group(1))


def _layer(cout=64, cin=128, T=32, base=0x10000000):
    p = lambda k: base + 0x100000 * k   # fake, 16-byte aligned device addresses (never dereferenced)
    return b.LcpLayer(p(1), p(2), p(3), p(4), p(5), p(6), None, None, cout, cin, T)


def _ws(layers, hp):
    arr = (b.LcpLayer * len(layers))(*layers)
    n = ctypes.c_size_t(0)
    st = b.lib().lcp_workspace_size(arr, len(layers), ctypes.byref(hp), ctypes.byref(n))
    return st, n.value


def test_workspace_size_for_valid_layers():
    hp = b.hparams(64, 2, 4, 5, 0.5, b.BF16)
    st, n = _ws([_layer()], hp)
    assert st == 0 and n > 0
    st2, n2 = _ws([_layer(), _layer(cout=128)], hp)
    assert st2 == 0 and n2 >= n
    st0, n0 = _ws([], hp)
    assert st0 == 0 and n0 == 0


@pytest.mark.parametrize("mut,code", [
    (lambda l, h: setattr(h, "block", 48), 2),
    (lambda l, h: setattr(h, "block", 512), 2),
    (lambda l, h: setattr(h, "m", 6), 2),
    (lambda l, h: setattr(h, "n", 0), 2),
    (lambda l, h: setattr(h, "n", 5), 2),
    (lambda l, h: setattr(h, "iters", 0), 7),
    (lambda l, h: setattr(h, "tau", 0.0), 7),
    (lambda l, h: setattr(h, "tau", float("inf")), 7),
    (lambda l, h: setattr(h, "dtype", 9), 3),
    (lambda l, h: setattr(h, "flags", 0x100), 7),
    (lambda l, h: setattr(l, "W", None), 1),
    (lambda l, h: setattr(l, "loss", None), 1),
    (lambda l, h: setattr(l, "cout", 12), 2),
    (lambda l, h: setattr(l, "cout", 0), 2),
    (lambda l, h: setattr(l, "cin", 96), 2),       # not a multiple of B = 64
    (lambda l, h: setattr(l, "tokens", 0), 2),
    (lambda l, h: setattr(l, "X", 0x10000008), 7),  # misaligned
    (lambda l, h: setattr(h, "flags", b.FLAG_WRITE_WPRIME), 1),  # needs layer.Wp
    (lambda l, h: setattr(h, "flags", b.FLAG_CACHED_DENSE), 1),  # needs layer.Yd
    (lambda l, h: (setattr(h, "flags", b.FLAG_CACHED_DENSE), setattr(l, "Yd", 0x10000004)), 7),  # misaligned
    (lambda l, h: setattr(h, "flags", b.FLAG_SCORE), 1),          # needs layer.S
    (lambda l, h: (setattr(h, "flags", b.FLAG_SCORE), setattr(l, "S", 0x30000000), setattr(h, "block", 128),
                   setattr(l, "cin", 256)), 7),                     # tensor-core score path: B <= 64
])
def test_host_validation_codes(mut, code):
    l = _layer()
    hp = b.hparams(64, 2, 4, 5, 0.5, b.BF16)
    mut(l, hp)
    st, _ = _ws([l], hp)
    assert st == code
    assert b.lib().lcp_last_error().decode() != ""


def test_step_rejects_small_or_misaligned_workspace_without_a_gpu():
    L = b.lib()
    hp = b.hparams(64, 2, 4, 5, 0.5, b.BF16)
    arr = (b.LcpLayer * 1)(_layer())
    _, need = _ws([_layer()], hp)
    assert L.lcp_step(arr, 1, ctypes.byref(hp), 0x20000000, need - 1, None) == 4
    assert L.lcp_step(arr, 1, ctypes.byref(hp), 0x20000010, need, None) == 4
    assert L.lcp_step(arr, 0, ctypes.byref(hp), None, 0, None) == 0   # no layers: a no-op


def test_standalone_entry_points_validate_before_launch():
    L = b.lib()
    assert L.lcp_sinkhorn_fwd(None, 0x1000, None, 1, 64, 1.0, 5, None) == 1
    assert L.lcp_sinkhorn_fwd(0x1000, 0x2000, None, 1, 40, 1.0, 5, None) == 2
    assert L.lcp_sinkhorn_fwd(0x1000, 0x2000, None, 0, 64, 1.0, 5, None) == 0  # empty
    assert L.nm_mask(0x1000, 0x2000, 4, 30, 2, 4, 0, None) == 2
    assert L.nm_mask(0x1000, 0x2000, 4, 32, 2, 5, 0, None) == 2
    assert L.nm_mask(0x1000, 0x2000, 0, 32, 2, 4, 0, None) == 0               # empty
    assert L.lcp_loss_fwd(0x1000, 0x2000, 0x3000, 0x4000, 12, 5, None) == 2
    assert L.lcp_sinkhorn_bwd(0x1000, 0x2000, 0x3000, 0, 0x4000, 1, 64, 1.0, 5, None) == 7


def test_inference_entry_points_validate_before_launch():
    L = b.lib()
    # pack: W, mask, values, meta required; C_in a multiple of 32 and of B; B in {32, 64, 128, 256}
    assert L.lcp_pack24(None, 0x1000, 0x2000, 0x3000, 0x4000, 8, 128, 64, 1, None) == 1
    assert L.lcp_pack24(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 8, 100, 64, 1, None) == 2
    assert L.lcp_pack24(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 8, 128, 48, 1, None) == 2
    assert L.lcp_pack24(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 8, 96, 64, 1, None) == 2
    assert L.lcp_pack24(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 8, 128, 64, 9, None) == 3
    assert L.lcp_pack24(0x1008, 0x2000, 0x3000, 0x4000, 0x5000, 8, 128, 64, 1, None) == 7
    # gather: perm required, out of place, empty token count is a no-op
    assert L.lcp_gather(0x1000, None, 0x2000, 4, 128, 64, 1, None) == 1
    assert L.lcp_gather(0x1000, 0x3000, 0x1000, 4, 128, 64, 1, None) == 7
    assert L.lcp_gather(0x1000, 0x3000, 0x2000, 4, 128, 40, 1, None) == 2
    assert L.lcp_gather(0x1000, 0x3000, 0x2000, 0, 128, 64, 1, None) == 0
    # product: perm optional (B then unchecked), C_in too wide for one token's inputs
    assert L.lcp_sparse24_mm(0x1000, None, 0x2000, None, 0x3000, 8, 128, 4, 64, 1, None) == 1
    assert L.lcp_sparse24_mm(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 8, 128, 4, 40, 1, None) == 2
    assert L.lcp_sparse24_mm(0x1000, 0x2000, 0x3000, None, 0x5000, 8, 1 << 20, 1, 64, 1, None) == 2
    assert L.lcp_sparse24_mm(0x1000, 0x2000, 0x3000, None, 0x5000, 8, 128, 0, 0, 1, None) == 0
    # the widest rows whose one-token input image fits the 200 KB tile (bf16, float32)
    assert L.lcp_sparse24_mm(0x1000, 0x2000, 0x3000, None, 0x5000, 8, 91008 + 32, 1, 0, 1, None) == 2
    assert L.lcp_sparse24_mm(0x1000, 0x2000, 0x3000, None, 0x5000, 8, 91008, 1, 0, 1, None) != 2
    assert L.lcp_sparse24_mm(0x1000, 0x2000, 0x3000, None, 0x5000, 8, 48160 + 32, 1, 0, 0, None) == 2
    assert L.lcp_sparse24_mm(0x1000, 0x2000, 0x3000, None, 0x5000, 8, 48160, 1, 0, 0, None) != 2


def test_launch_count_reported():
    hp = b.hparams(64, 2, 4, 5, 0.5, b.F32)
    arr = (b.LcpLayer * 2)(_layer(), _layer())
    c = ctypes.c_int(0)
    assert b.lib().lcp_step_launches(arr, 2, ctypes.byref(hp), ctypes.byref(c)) == 0
    assert c.value > 0 and c.value % 2 == 0


def test_workspace_shrinks_when_the_caller_holds_yd():
    """A caller-provided Y_d replaces the workspace copy (T x C_out float32)."""
    hp = b.hparams(64, 2, 4, 5, 0.5, b.BF16)
    st, n = _ws([_layer(cout=256, T=512)], hp)
    l = _layer(cout=256, T=512)
    l.Yd = 0x70000000
    st2, n2 = _ws([l], hp)
    assert st == 0 and st2 == 0 and n - n2 >= 512 * 256 * 4


def test_adamw_and_train_validation():
    """Argument checks of lcp_adamw and lcp_train (host side, no launch)."""
    L = b.lib()
    opt = b.adamw_params()
    a = 0x10000000
    assert L.lcp_adamw(None, a, a, a, 64, ctypes.byref(opt), 1, None) == 1
    assert L.lcp_adamw(a, a, a, a, 62, ctypes.byref(opt), 1, None) == 2      # not a multiple of 4
    assert L.lcp_adamw(a, a, a, a, 64, ctypes.byref(opt), 0, None) == 7      # t < 1
    bad = b.adamw_params(beta2=1.0)
    assert L.lcp_adamw(a, a, a, a, 64, ctypes.byref(bad), 1, None) == 7
    assert L.lcp_adamw(a, a, a, a, 0, ctypes.byref(opt), 1, None) == 0       # empty: no-op
    hp = b.hparams(64, 2, 4, 5, 0.5, b.BF16)
    arr = (b.LcpLayer * 1)(_layer())
    st = (b.LcpAdamwState * 1)(b.LcpAdamwState(a, a))
    call = lambda first, count, total, t0=1.0, t1=0.1, state=st: L.lcp_train(
        arr, 1, ctypes.byref(hp), ctypes.byref(opt), state, first, count, total, t0, t1, a, 1 << 30, None)
    assert call(0, 5, 4) == 7            # beyond the run
    assert call(0, 1, 0) == 7            # empty run
    assert call(0, 1, 4, t1=0.0) == 7    # temperature must be positive
    assert call(0, 1, 4, state=None) == 1
    assert L.lcp_train(arr, 1, ctypes.byref(hp), None, st, 0, 1, 4, 1.0, 0.1, a, 1 << 30, None) == 1

"""Python binding of liblcp (ctypes): argument marshalling only.

Every operation runs in the CUDA library ``csrc/liblcp.so``; this module turns
torch tensors into device pointers and the current torch stream into a
``cudaStream_t``.  PyTorch is used for device memory and streams only.  If the
library is missing, the first call raises: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc", "liblcp.so")

F32, BF16 = 0, 1
FLAG_WRITE_WPRIME = 0x1
FLAG_SIMT = 0x2
FLAG_CACHED_DENSE = 0x4
FLAG_HARD = 0x8
FLAG_SCORE = 0x10
SCORE_MAGNITUDE, SCORE_WANDA, SCORE_RIA = 0, 1, 2
TIMED_EVENTS = 8
STAGES = ("sinkhorn_fwd", "permute_mask", "calib_gemm", "loss", "bwd_gemm", "block_bwd", "sinkhorn_bwd")

_c_void_p, _c_int, _c_float = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


class LcpLayer(ctypes.Structure):
    _fields_ = [("W", _c_void_p), ("X", _c_void_p), ("L", _c_void_p), ("P", _c_void_p),
                ("dL", _c_void_p), ("loss", _c_void_p), ("mask", _c_void_p), ("Wp", _c_void_p),
                ("cout", _c_int), ("cin", _c_int), ("tokens", _c_int), ("Yd", _c_void_p), ("perm", _c_void_p),
                ("S", _c_void_p)]


class LcpHparams(ctypes.Structure):
    _fields_ = [("block", _c_int), ("n", _c_int), ("m", _c_int), ("iters", _c_int), ("tau", _c_float),
                ("dtype", _c_int), ("flags", ctypes.c_uint)]


class LcpAdamwParams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double), ("beta2", ctypes.c_double),
                ("eps", ctypes.c_double), ("weight_decay", ctypes.c_double)]


class LcpAdamwState(ctypes.Structure):
    _fields_ = [("m", _c_void_p), ("v", _c_void_p)]


class LcpError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load liblcp.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                           "`python -m learnable_channel_permutation_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    sig = {
        "lcp_abi_version": ([], _c_int),
        "lcp_last_error": ([], ctypes.c_char_p),
        "lcp_status_string": ([_c_int], ctypes.c_char_p),
        "lcp_workspace_size": ([P(LcpLayer), _c_int, P(LcpHparams), P(ctypes.c_size_t)], _c_int),
        "lcp_step_launches": ([P(LcpLayer), _c_int, P(LcpHparams), P(_c_int)], _c_int),
        "lcp_step": ([P(LcpLayer), _c_int, P(LcpHparams), _c_void_p, ctypes.c_size_t, _c_void_p], _c_int),
        "lcp_step_timed": ([P(LcpLayer), _c_int, P(LcpHparams), _c_void_p, ctypes.c_size_t, _c_void_p,
                            P(_c_void_p), _c_int], _c_int),
        "lcp_step_shard": ([P(LcpLayer), _c_int, P(LcpHparams), _c_int, P(_c_void_p), P(_c_void_p), _c_void_p,
                            ctypes.c_size_t, _c_void_p], _c_int),
        "lcp_sinkhorn_fwd": ([_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_float, _c_int, _c_void_p], _c_int),
        "lcp_sinkhorn_bwd": ([_c_void_p, _c_void_p, _c_void_p, _c_int, _c_void_p, _c_int, _c_int, _c_float,
                              _c_int, _c_void_p], _c_int),
        "lcp_permute_weight": ([_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_void_p], _c_int),
        "nm_mask": ([_c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_void_p], _c_int),
        "lcp_loss_fwd": ([_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_void_p], _c_int),
        "lcp_loss_bwd": ([_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_void_p], _c_int),
        "lcp_loss_fwd_static": ([_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_void_p], _c_int),
        "lcp_calib_gemm": ([_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int,
                            _c_void_p], _c_int),
        "lcp_grad_gemm": ([_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_void_p], _c_int),
        "lcp_calib_gemm_loss": ([_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int,
                                 _c_int, _c_void_p], _c_int),
        "lcp_loss_pair": ([_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int,
                           _c_int, _c_void_p], _c_int),
        "lcp_device_error": ([P(_c_int), _c_int], _c_int),
        "lcp_harden": ([_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_void_p], _c_int),
        "lcp_score": ([_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_int,
                       _c_void_p], _c_int),
        "lcp_adamw": ([_c_void_p, _c_void_p, _c_void_p, _c_void_p, ctypes.c_longlong, P(LcpAdamwParams), _c_int,
                       _c_void_p], _c_int),
        "lcp_train": ([P(LcpLayer), _c_int, P(LcpHparams), P(LcpAdamwParams), P(LcpAdamwState), _c_int, _c_int,
                       _c_int, _c_float, _c_float, _c_void_p, ctypes.c_size_t, _c_void_p], _c_int),
        "lcp_selftest_bounded_wait": ([P(_c_int)], _c_int),
        "lcp_pack24": ([_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int,
                        _c_void_p], _c_int),
        "lcp_gather": ([_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_void_p], _c_int),
        "lcp_sparse24_mm": ([_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int,
                             _c_int, _c_void_p], _c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def check(status: int) -> None:
    if status != 0:
        L = lib()
        raise LcpError(status, f"{L.lcp_status_string(status).decode()} -- {L.lcp_last_error().decode()}")


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor], dtype=None, name: str = "") -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def hparams(block: int, n: int, m: int, iters: int, tau: float, dtype: int, flags: int = 0) -> LcpHparams:
    return LcpHparams(block, n, m, iters, float(tau), dtype, flags)


def make_layer(d: Dict[str, torch.Tensor], wdtype) -> LcpLayer:
    W, X, Lg = d["W"], d["X"], d["L"]
    cout, cin = W.shape
    tokens = X.shape[0]
    if X.shape[1] != cin:
        raise ValueError("X must be [T, C_in]")
    return LcpLayer(_ptr(W, wdtype, "W"), _ptr(X, wdtype, "X"), _ptr(Lg, torch.float32, "L"),
                    _ptr(d["P"], torch.float32, "P"), _ptr(d["dL"], torch.float32, "dL"),
                    _ptr(d["loss"], torch.float32, "loss"), _ptr(d.get("mask"), torch.int32, "mask"),
                    _ptr(d.get("Wp"), torch.float32, "Wp"), cout, cin, tokens,
                    _ptr(d.get("Yd"), torch.float32, "Yd"), _ptr(d.get("perm"), torch.int32, "perm"),
                    _ptr(d.get("S"), wdtype, "S"))


class Step:
    """A prepared lcp_step call: the layer descriptors, hyper-parameters and
    workspace are marshalled once; ``run()`` enqueues one step on a stream."""

    def __init__(self, layers: Sequence[Dict[str, torch.Tensor]], block: int, n: int, m: int, iters: int,
                 tau: float, flags: int = 0, workspace: Optional[torch.Tensor] = None):
        if not layers:
            raise ValueError("at least one layer")
        wdtype = layers[0]["W"].dtype
        self.hp = hparams(block, n, m, iters, tau, _dt(layers[0]["W"]), flags)
        self.arr = (LcpLayer * len(layers))(*[make_layer(d, wdtype) for d in layers])
        self.n = len(layers)
        self.layers = list(layers)  # keep the tensors alive
        nbytes = ctypes.c_size_t(0)
        check(lib().lcp_workspace_size(self.arr, self.n, ctypes.byref(self.hp), ctypes.byref(nbytes)))
        self.ws_bytes = int(nbytes.value)
        if workspace is None:
            workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=layers[0]["W"].device)
        if workspace.numel() < self.ws_bytes:
            raise ValueError("workspace too small")
        self.ws = workspace
        c = _c_int(0)
        check(lib().lcp_step_launches(self.arr, self.n, ctypes.byref(self.hp), ctypes.byref(c)))
        self.launches = int(c.value)

    def run(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        check(lib().lcp_step(self.arr, self.n, ctypes.byref(self.hp), self.ws.data_ptr(), self.ws.numel(),
                             _stream(stream)))

    def run_timed(self, events: List[torch.cuda.Event], stream: Optional[torch.cuda.Stream] = None) -> None:
        """Stage events of the first layer (TIMED_EVENTS events) or of every
        layer (TIMED_EVENTS per layer, layer by layer)."""
        if len(events) not in (TIMED_EVENTS, TIMED_EVENTS * self.n):
            raise ValueError(f"need {TIMED_EVENTS} or {TIMED_EVENTS} x {self.n} events")
        for e in events:
            if e.cuda_event == 0:
                raise ValueError("events must be created (record once) before use")
        arr = (_c_void_p * len(events))(*[e.cuda_event for e in events])
        check(lib().lcp_step_timed(self.arr, self.n, ctypes.byref(self.hp), self.ws.data_ptr(), self.ws.numel(),
                                   _stream(stream), arr, len(events)))


def step_shard(step: "Step", total_tokens: int, dP: Sequence[torch.Tensor], ckpt: Sequence[torch.Tensor],
               stream: Optional[torch.cuda.Stream] = None) -> None:
    """lcp_step_shard on a prepared Step whose layers hold one token shard:
    dP[i] and ckpt[i] receive layer i's shard gradient d loss / d P and its
    Sinkhorn checkpoint; the losses are normalised by ``total_tokens``."""
    if len(dP) != step.n or len(ckpt) != step.n:
        raise ValueError("one dP and one ckpt tensor per layer")
    dps = (_c_void_p * step.n)(*[_ptr(t, torch.float32, "dP") for t in dP])
    cks = (_c_void_p * step.n)(*[_ptr(t, torch.float32, "ckpt") for t in ckpt])
    check(lib().lcp_step_shard(step.arr, step.n, ctypes.byref(step.hp), int(total_tokens), dps, cks,
                               step.ws.data_ptr(), step.ws.numel(), _stream(stream)))


def adamw_params(lr: float = 1e-3, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
                 weight_decay: float = 0.01) -> LcpAdamwParams:
    return LcpAdamwParams(lr, beta1, beta2, eps, weight_decay)


def adamw(L: torch.Tensor, dL: torch.Tensor, m: torch.Tensor, v: torch.Tensor, opt: LcpAdamwParams, t: int) -> None:
    check(lib().lcp_adamw(_ptr(L, torch.float32, "L"), _ptr(dL, torch.float32, "dL"), _ptr(m, torch.float32, "m"),
                          _ptr(v, torch.float32, "v"), L.numel(), ctypes.byref(opt), t, _stream(None)))


class Trainer:
    """AdamW training of the logits of prepared layers (lcp_train): ``run(first,
    count)`` enqueues steps first .. first + count - 1 of a ``total``-step run
    with the temperature going linearly from ``tau_start`` to ``tau_end``."""

    def __init__(self, step: "Step", opt: LcpAdamwParams, total: int, tau_start: float = 1.0,
                 tau_end: float = 0.1):
        self.step, self.opt, self.total = step, opt, total
        self.tau_start, self.tau_end = tau_start, tau_end
        self.moments = [(torch.zeros_like(d["L"]), torch.zeros_like(d["L"])) for d in step.layers]
        self.state = (LcpAdamwState * len(self.moments))(*[LcpAdamwState(m.data_ptr(), v.data_ptr())
                                                           for m, v in self.moments])

    def run(self, first: int, count: int, stream: Optional[torch.cuda.Stream] = None) -> None:
        s = self.step
        check(lib().lcp_train(s.arr, s.n, ctypes.byref(s.hp), ctypes.byref(self.opt), self.state, first, count,
                              self.total, self.tau_start, self.tau_end, s.ws.data_ptr(), s.ws.numel(),
                              _stream(stream)))


def capture(step: "Step", events: Optional[List[torch.cuda.Event]] = None) -> "torch.cuda.CUDAGraph":
    """Capture one lcp_step (and, with ``events``, its stage events) into a CUDA
    graph; replaying it re-runs the step on the same buffers with one launch."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step.run(side)                     # first call outside capture (one-time set-up)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        if events is None:
            step.run()
        else:
            step.run_timed(events)
    return g


def alloc_outputs(W: torch.Tensor, X: torch.Tensor, L: torch.Tensor, with_mask: bool = True,
                  with_wp: bool = False) -> Dict[str, torch.Tensor]:
    dev = W.device
    cout, cin = W.shape
    d = dict(W=W, X=X, L=L, P=torch.empty_like(L), dL=torch.empty_like(L),
             loss=torch.empty(4, dtype=torch.float32, device=dev))
    if with_mask:
        d["mask"] = torch.empty(cout, cin // 32, dtype=torch.int32, device=dev)
    if with_wp:
        d["Wp"] = torch.empty(cout, cin, dtype=torch.float32, device=dev)
    return d


def step(layers: Sequence[Dict[str, torch.Tensor]], block: int, n: int, m: int, iters: int, tau: float,
         flags: int = 0) -> Step:
    """Run one forward+backward step on the current stream (allocates a workspace)."""
    s = Step(layers, block, n, m, iters, tau, flags)
    s.run()
    return s


def sinkhorn_fwd(L: torch.Tensor, P: torch.Tensor, ckpt: Optional[torch.Tensor], tau: float, iters: int) -> None:
    nb, B, _ = L.shape
    check(lib().lcp_sinkhorn_fwd(_ptr(L, torch.float32, "L"), _ptr(P, torch.float32, "P"),
                                 _ptr(ckpt, torch.float32, "ckpt"), nb, B, float(tau), iters, _stream(None)))


def sinkhorn_bwd(L: torch.Tensor, ckpt: torch.Tensor, dP: torch.Tensor, dL: torch.Tensor, tau: float,
                 iters: int) -> None:
    nb, B, _ = L.shape
    splits = dP.numel() // (nb * B * B)
    check(lib().lcp_sinkhorn_bwd(_ptr(L, torch.float32, "L"), _ptr(ckpt, torch.float32, "ckpt"),
                                 _ptr(dP, torch.float32, "dP"), splits, _ptr(dL, torch.float32, "dL"), nb, B,
                                 float(tau), iters, _stream(None)))


def permute_weight(W: torch.Tensor, P: torch.Tensor, Wp: torch.Tensor) -> None:
    cout, cin = W.shape
    check(lib().lcp_permute_weight(_ptr(W, None, "W"), _ptr(P, torch.float32, "P"), _ptr(Wp, torch.float32, "Wp"),
                                   cout, cin, P.shape[1], _dt(W), _stream(None)))


def score(W: torch.Tensor, X: torch.Tensor, kind: int) -> torch.Tensor:
    """Importance scores S of W (LCP_SCORE_*), in W's dtype."""
    cout, cin = W.shape
    S = torch.empty_like(W)
    stats = torch.empty(2 * cin + cout, dtype=torch.float32, device=W.device)
    check(lib().lcp_score(_ptr(W, None, "W"), _ptr(X, W.dtype, "X"), _ptr(S, W.dtype, "S"),
                          _ptr(stats, torch.float32, "stats"), cout, cin, X.shape[0], kind, _dt(W), _stream(None)))
    return S


def harden(P: torch.Tensor, perm: torch.Tensor, P_hard: Optional[torch.Tensor] = None) -> None:
    nb, B, _ = P.shape
    check(lib().lcp_harden(_ptr(P, torch.float32, "P"), _ptr(perm, torch.int32, "perm"),
                           _ptr(P_hard, torch.float32, "P_hard"), nb, B, _stream(None)))


def nm_mask(Wp: torch.Tensor, bits: torch.Tensor, n: int, m: int) -> None:
    rows, cols = Wp.shape
    check(lib().nm_mask(_ptr(Wp, None, "Wp"), _ptr(bits, torch.int32, "bits"), rows, cols, n, m, _dt(Wp),
                        _stream(None)))


def pack24(W: torch.Tensor, perm: Optional[torch.Tensor], mask_bits: torch.Tensor, block: int):
    """Compressed 2:4 weight (values [C_out, C_in/2] in W's dtype, meta [C_out, C_in/32]
    int32 words) of A = M.(W P_B) for the hard permutation perm [C_in/B, B]."""
    cout, cin = W.shape
    vals = torch.empty(cout, cin // 2, dtype=W.dtype, device=W.device)
    meta = torch.empty(cout, cin // 32, dtype=torch.int32, device=W.device)
    check(lib().lcp_pack24(_ptr(W, None, "W"), _ptr(perm, torch.int32, "perm"), _ptr(mask_bits, torch.int32, "mask"),
                           _ptr(vals, W.dtype, "values"), _ptr(meta, torch.int32, "meta"), cout, cin, block, _dt(W),
                           _stream(None)))
    return vals, meta


def gather(X: torch.Tensor, perm: torch.Tensor, Xp: Optional[torch.Tensor] = None) -> torch.Tensor:
    """x_pi = P_B^T x for every token row of X [T, C_in]."""
    T, cin = X.shape
    Xp = torch.empty_like(X) if Xp is None else Xp
    check(lib().lcp_gather(_ptr(X, None, "X"), _ptr(perm, torch.int32, "perm"), _ptr(Xp, X.dtype, "Xp"), T, cin,
                           perm.shape[1], _dt(X), _stream(None)))
    return Xp


def sparse24_mm(vals: torch.Tensor, meta: torch.Tensor, X: torch.Tensor, perm: Optional[torch.Tensor],
                block: int, Y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y [T, C_out] float32 = x_pi A^T from the compressed weight (perm None: X already permuted)."""
    T, cin = X.shape
    cout = vals.shape[0]
    Y = torch.empty(T, cout, dtype=torch.float32, device=X.device) if Y is None else Y
    check(lib().lcp_sparse24_mm(_ptr(vals, X.dtype, "values"), _ptr(meta, torch.int32, "meta"), _ptr(X, None, "X"),
                                _ptr(perm, torch.int32, "perm"), _ptr(Y, torch.float32, "Y"), cout, cin, T, block,
                                _dt(X), _stream(None)))
    return Y


def calib_gemm(X: torch.Tensor, W: torch.Tensor, At: Optional[torch.Tensor], Yd: torch.Tensor,
               Ys: Optional[torch.Tensor]) -> None:
    T, cin = X.shape
    cout = W.shape[0]
    bf = torch.bfloat16
    check(lib().lcp_calib_gemm(_ptr(X, bf, "X"), _ptr(W, bf, "W"), _ptr(At, bf, "At"),
                               _ptr(Yd, torch.float32, "Yd"), _ptr(Ys, torch.float32, "Ys"), T, cout, cin,
                               _stream(None)))


def calib_gemm_loss(X: torch.Tensor, W: torch.Tensor, At: torch.Tensor, D: torch.Tensor, Ys: torch.Tensor,
                    partials: torch.Tensor) -> None:
    """lcp_calib_gemm_loss: D = Y_d - Y_s and Y_s (bf16 [T, C_out]) and the
    per-token slot partials (float32 [T, ceil(C_out/64), 4])."""
    T, cin = X.shape
    cout = W.shape[0]
    bf = torch.bfloat16
    check(lib().lcp_calib_gemm_loss(_ptr(X, bf, "X"), _ptr(W, bf, "W"), _ptr(At, bf, "At"), _ptr(D, bf, "D"),
                                    _ptr(Ys, bf, "Ys"), _ptr(partials, torch.float32, "partials"), T, cout, cin,
                                    _stream(None)))


def loss_pair(D: torch.Tensor, Ys: torch.Tensor, partials: torch.Tensor, loss: torch.Tensor, stats: torch.Tensor,
              G: torch.Tensor, counter: torch.Tensor) -> None:
    """lcp_loss_pair: the loss and G (bf16) from lcp_calib_gemm_loss's outputs;
    ``counter`` is one int32 of device memory, zero before the call."""
    T, cout = D.shape
    bf = torch.bfloat16
    check(lib().lcp_loss_pair(_ptr(D, bf, "D"), _ptr(Ys, bf, "Ys"), _ptr(partials, torch.float32, "partials"),
                              _ptr(loss, torch.float32, "loss"), _ptr(stats, torch.float32, "stats"), _ptr(G, bf, "G"),
                              _ptr(counter, torch.int32, "counter"), cout, T, _stream(None)))


def grad_gemm(G: torch.Tensor, X: torch.Tensor, dAt: torch.Tensor) -> None:
    T, cout = G.shape
    cin = X.shape[1]
    bf = torch.bfloat16
    check(lib().lcp_grad_gemm(_ptr(G, bf, "G"), _ptr(X, bf, "X"), _ptr(dAt, bf, "dAt"), T, cout, cin,
                              _stream(None)))


def selftest_bounded_wait() -> int:
    """Runs the bounded-wait self-test (about 2 s) and returns the recorded site (901)."""
    v = _c_int(0)
    check(lib().lcp_selftest_bounded_wait(ctypes.byref(v)))
    return v.value


def device_error(reset: bool = True) -> int:
    """Site code of the first tensor-core wait that expired (0 = none); synchronous."""
    v = _c_int(0)
    check(lib().lcp_device_error(ctypes.byref(v), 1 if reset else 0))
    return int(v.value)


def loss_fwd(Yd: torch.Tensor, Ys: torch.Tensor, loss: torch.Tensor, stats: torch.Tensor) -> None:
    T, cout = Yd.shape
    check(lib().lcp_loss_fwd(_ptr(Yd, torch.float32, "Yd"), _ptr(Ys, torch.float32, "Ys"),
                             _ptr(loss, torch.float32, "loss"), _ptr(stats, torch.float32, "stats"), cout, T,
                             _stream(None)))


def loss_bwd(Yd: torch.Tensor, Ys: torch.Tensor, stats: torch.Tensor, G: torch.Tensor) -> None:
    T, cout = Yd.shape
    check(lib().lcp_loss_bwd(_ptr(Yd, torch.float32, "Yd"), _ptr(Ys, torch.float32, "Ys"),
                             _ptr(stats, torch.float32, "stats"), _ptr(G, None, "G"), cout, T, _dt(G),
                             _stream(None)))


STATIC_MAX_TOKENS = 65536


def loss_fwd_static(Yd: torch.Tensor, Ys: torch.Tensor, loss: torch.Tensor) -> None:
    """lcp_loss_fwd without a scratch argument: for callers that cannot allocate
    device memory (see lcp_loss_fwd_static in include/lcp.h)."""
    T, cout = Yd.shape
    check(lib().lcp_loss_fwd_static(_ptr(Yd, torch.float32, "Yd"), _ptr(Ys, torch.float32, "Ys"),
                                    _ptr(loss, torch.float32, "loss"), cout, T, _stream(None)))

#!/usr/bin/env python
"""Benchmark of the learnable-channel-permutation forward+backward step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One "step" is one pass of the whole hot path (Sinkhorn, permutation + N:M
mask, dense and sparse calibration outputs, cosine loss, backward to the
logits) over one layer.  The default workload is a LLaMA-7B q_proj-shaped
layer: W 4096x4096 bf16 with 1% outlier input channels, T = 2048 calibration
tokens, B = 64, 2:4, tau = 0.5, 5 Sinkhorn iterations (seeded synthetic data).

Multi-GPU (torchrun): every rank runs its own independent layer (distinct
seed): the work is sharded by layer, with no collective on the data path;
``value`` is the total number of layer-steps per second over all ranks,
timed as the maximum over ranks (weak scaling).

Timing: W untimed warm-up steps, then K steps, each timed with CUDA events
on the launching stream; the L2 cache is flushed (a 256 MiB write) between
timed steps, outside the events.  Per-kernel durations come from events the
library records between its stages inside the same timed steps.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LCP fwd+bwd steps/s per layer @4096x4096 B=64 2:4; % of bf16 TC peak & HBM BW"
UNIT = "steps/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload(name):
    from learnable_channel_permutation_b200 import synth
    if name == "q_proj_4096":
        return synth.q_proj_4096()
    if name == "toy_256":
        return synth.toy_256()
    if name in ("sweep_4096_b128", "sweep_4096_b256"):
        # the sweep's 4096 x 4096 layer (T = 2048) at B = 128 / 256, 5 iterations, tau 1.0, 2:4
        return synth.sweep_4096(int(name[-3:]), 5, 1.0, 2, 4)
    raise SystemExit(f"unknown workload {name}")


def stage_work(wl, li, splits=1, fused_loss=True):
    """Algorithmic work of each stage for one layer: (kind, amount).

    kind "flop" for the tensor-core contractions, "byte" for the HBM-bound
    stages (compulsory bytes: every input read once, every output written once).
    With the loss reduction in the calibration GEMM's epilogue (the bf16
    tensor-core path) the loss stage reads D and Y_s in bf16 and the slot
    partials; otherwise Y_d and Y_s in float32.
    """
    co, ci, T = li.spec.cout, li.spec.cin, li.spec.tokens
    B, it = wl.block, wl.iters
    nb = ci // B
    e = 2 if wl.dtype == "bf16" else 4
    loss_bytes = (T * co * (2 + 2 + e) + T * ((co + 63) // 64) * 16 + T * 16 if fused_loss
                  else T * co * (4 + 4 + e) + T * 16)
    return {
        "sinkhorn_fwd": ("byte", nb * B * B * (4 + 4 + 3 * 2) + nb * it * 2 * B * 4),
        "permute_mask": ("byte", co * ci * (e + e) + co * ci // 8 + 3 * nb * B * B * 2),
        "calib_gemm": ("flop", 2 * 2 * T * co * ci),
        "loss": ("byte", loss_bytes),
        "bwd_gemm": ("flop", 2 * T * co * ci),
        "block_bwd": ("byte", co * ci * (e + e) + co * ci // 8 + splits * nb * B * B * 4),
        "sinkhorn_bwd": ("byte", nb * B * B * (4 + 4 * splits + 4) + nb * it * 2 * B * 4),
    }


def src_hash(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
            if self.uuid:
                cmd.insert(1, f"--id={self.uuid}")
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        # median over samples taken while the GPU was busy (above half of max)
        busy = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": float(np.median(busy)) if busy else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def cpu_baseline(wl, budget_s=12.0):
    """Time the CPU oracle (as it stands) on whole steps of the same workload."""
    from oracle import lcp_oracle as O
    from learnable_channel_permutation_b200 import synth
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count()
    li = synth.make_inputs(wl)[0]
    n, t0 = 0, time.perf_counter()
    while True:
        O.step(li.W, li.X, li.L, wl.tau, wl.iters, wl.n, wl.m)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 20:
            break
    return {"value": n / el, "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "sample": f"{n} whole fwd+bwd steps of the {wl.name} layer (float64 numpy oracle, "
                      f"BLAS threads = {cores}), {el:.1f} s"}


def reference_arm(args, rank, world):
    """The oracle timed on the host cores (only rank 0 works under torchrun):
    W untimed and K timed whole fwd+bwd steps of the workload's layer."""
    from oracle import lcp_oracle as O
    from learnable_channel_permutation_b200 import synth
    if rank != 0:
        return 0
    wl = workload(args.workload)
    li = synth.make_inputs(wl)[0]
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count()
    for _ in range(max(args.warmup, 0)):
        O.step(li.W, li.X, li.L, wl.tau, wl.iters, wl.n, wl.m)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.step(li.W, li.X, li.L, wl.tau, wl.iters, wl.n, wl.m)
    el = time.perf_counter() - t0
    value = args.steps / el
    sample = (f"{args.steps} whole fwd+bwd steps of the {wl.name} layer (T={li.spec.tokens}) timed after "
              f"{args.warmup} untimed ones, {el:.1f} s; float64 numpy oracle, BLAS threads = {cores}")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
            "config": {"workload": wl.name, "cout": li.spec.cout, "cin": li.spec.cin, "tokens": li.spec.tokens,
                       "block": wl.block, "nm": f"{wl.n}:{wl.m}", "tau": wl.tau, "iters": wl.iters},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(cores), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="q_proj_4096")
    ap.add_argument("--simt", action="store_true", help="CUDA-core kernels for every contraction")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of CUDA-graph replays")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the secondary measurements (cached dense output, standalone mask, "
                         "Sinkhorn scaling run, one-core oracle)")
    ap.add_argument("--only-extra", default=None,
                    choices=["cached_dense", "hard_step", "score_step", "train", "cublas_same_products", "configs",
                             "inference_24", "nm_mask", "sinkhorn_scaling", "stream_ref"],
                    help="run this one secondary measurement only")
    ap.add_argument("--scaling-blocks", type=int, default=40 * (6 * 5120 + 13824) // 64,
                    help="64 x 64 blocks of the Sinkhorn scaling run (default: every projection of a "
                         "40-layer 13B-shaped model, 27 840 blocks)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return reference_arm(args, rank, world)

    import torch
    import torch.distributed as dist
    from learnable_channel_permutation_b200 import binding as b
    from learnable_channel_permutation_b200 import synth

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    from learnable_channel_permutation_b200 import parallel
    wl = parallel.rank_workload(workload(args.workload), rank)   # each rank: its own layer
    li = synth.make_inputs(wl)[0]
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    W = torch.from_numpy(li.W).to(dev).to(tdt)
    X = torch.from_numpy(li.X).to(dev).to(tdt)
    L = torch.from_numpy(li.L).to(dev)
    layer = b.alloc_outputs(W, X, L)
    flags = b.FLAG_SIMT if args.simt else 0
    step = b.Step([layer], wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=flags)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    K = args.steps
    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    uuid = f"GPU-{uuid}" if uuid and not str(uuid).startswith("GPU-") else (str(uuid) if uuid else None)
    sampler = ClockSampler(uuid if world == 1 else None)

    def time_steps(run_one):
        """W warm-up calls, then K timed ones with L2 flushed before each; the
        device time between events recorded right before and after each call."""
        for _ in range(args.warmup):
            run_one()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        for k in range(K):
            flush.zero_()                      # L2 flush, outside the timed events
            e0[k].record()
            run_one()
            e1[k].record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return sum(e0[k].elapsed_time(e1[k]) for k in range(K))

    def stage_breakdown():
        """Per-stage averages from a graph that also records the stage events
        (an event between two kernels keeps the second from starting early, so
        these stages add up to a little more than the headline step time)."""
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(b.TIMED_EVENTS)]
        for e in ev:
            e.record()
        g = b.capture(step, ev)
        for _ in range(args.warmup):
            g.replay()
        rows = []
        for _ in range(K):
            flush.zero_()
            g.replay()
            torch.cuda.synchronize()           # the stage events are reused by every replay
            rows.append([ev[s].elapsed_time(ev[s + 1]) for s in range(len(b.STAGES))])
        del g
        return {name: sum(r[i] for r in rows) / K for i, name in enumerate(b.STAGES)}

    graph_mode = not args.eager
    sampler.start()
    time.sleep(0.2)
    if graph_mode:
        g_step = b.capture(step)
        total_ms = time_steps(g_step.replay)
    else:
        total_ms = time_steps(step.run)
    clocks = sampler.stop()
    eager_total = time_steps(step.run) if graph_mode else None
    if graph_mode:
        del g_step
    stage_ms = stage_breakdown()

    max_ms, max_eager = parallel.max_over_ranks([total_ms, eager_total or 0.0], device=dev)
    value = parallel.job_throughput(K, world, max_ms)
    eager = None
    if eager_total is not None:
        eager = {"value": parallel.job_throughput(K, world, max_eager), "ms_per_step": max_eager / K}

    # End to end through the public API, a 2-deep pipeline: two device input sets
    # on a copy stream keep the host-to-device copy of step k + 1 in flight while
    # step k computes; the time runs from the first copy to the last read-back.
    # `e2e`: a training loop's traffic -- every step brings its calibration tokens
    # X from pinned host memory (the layer's W and logits L stay on the device as
    # its state) and reads its loss back.  `e2e_all_inputs`: every step copies W,
    # X and L in and reads loss and dL back.
    e2e = e2e_all = None
    if not args.no_e2e:
        hW = torch.from_numpy(li.W).to(tdt).pin_memory()
        hX = torch.from_numpy(li.X).to(tdt).pin_memory()
        hL = torch.from_numpy(li.L).pin_memory()
        hloss = torch.empty(4, dtype=torch.float32).pin_memory()
        hdL = torch.empty_like(hL).pin_memory()
        layer2 = b.alloc_outputs(W.clone(), torch.empty_like(X), L.clone())
        sets = [layer, layer2]
        steps = [step, b.Step([layer2], wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=flags, workspace=step.ws)]
        cstream = torch.cuda.Stream()

        def measure(all_inputs):
            copied = [torch.cuda.Event(), torch.cuda.Event()]
            freed = [torch.cuda.Event(), torch.cuda.Event()]

            def issue(k):
                j = k % 2
                with torch.cuda.stream(cstream):
                    if k >= 2:
                        cstream.wait_event(freed[j])          # step k - 2 is done with input set j
                    if all_inputs:
                        sets[j]["W"].copy_(hW, non_blocking=True)
                        sets[j]["L"].copy_(hL, non_blocking=True)
                    sets[j]["X"].copy_(hX, non_blocking=True)
                    copied[j].record(cstream)
                stream.wait_event(copied[j])
                steps[j].run(stream)
                hloss[:1].copy_(sets[j]["loss"][:1], non_blocking=True)
                if all_inputs:
                    hdL.copy_(sets[j]["dL"], non_blocking=True)
                freed[j].record(stream)

            Ke = max(4, min(K, 20))
            for k in range(2):
                issue(k)
            torch.cuda.synchronize()
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(cstream)
            for k in range(Ke):
                issue(k)
            t1.record(stream)
            torch.cuda.synchronize()
            (te_ms,) = parallel.max_over_ranks([t0.elapsed_time(t1) / Ke], device=dev)
            h2d = hX.numel() * hX.element_size()
            d2h = 4
            if all_inputs:
                h2d += hW.numel() * hW.element_size() + hL.numel() * 4
                d2h += hdL.numel() * 4
            return {"value": parallel.job_throughput(1, world, te_ms), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h), "steps": Ke,
                    "pipeline": "2 input sets: step k+1's host-to-device copy overlaps step k"}

        e2e = measure(False)
        e2e["inputs"] = ("per step: the step's calibration tokens X host-to-device (W and L stay on the "
                         "device as the layer's state), the loss device-to-host")
        e2e_all = measure(True)
        e2e_all["inputs"] = "per step: W, X and L host-to-device, loss and dL device-to-host"

    if world > 1:
        dist.barrier()
    if rank != 0:
        dist.destroy_process_group()
        return 0

    pk, pk_src = peaks()
    work = stage_work(wl, li, fused_loss=wl.dtype == "bf16" and not args.simt)
    dom = max(stage_ms, key=lambda s: stage_ms[s])
    kind, amount = work[dom]
    dur_s = stage_ms[dom] / 1e3
    if kind == "flop":
        achieved = amount / dur_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_tflops"]}
    else:
        achieved = amount / dur_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"]}
    roof.update({"kernel": dom, "peak_source": f"{pk_src} ({'bf16 burst' if kind == 'flop' else 'copy'})",
                 "traffic": traffic_for(dom, args.simt), "algorithmic": amount,
                 "algorithmic_unit": "FLOP" if kind == "flop" else "bytes"})
    per_stage = {}
    for s in b.STAGES:
        kd, am = work[s]
        ms = stage_ms[s]
        if kd == "flop":
            per_stage[s] = {"ms": ms, "TFLOP/s": am / (ms / 1e3) / 1e12,
                            "frac": am / (ms / 1e3) / 1e12 / pk["bf16_tflops"]}
        else:
            per_stage[s] = {"ms": ms, "GB/s": am / (ms / 1e3) / 1e9, "frac": am / (ms / 1e3) / 1e9 / pk["hbm_gbs"]}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": max_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic (seeded)",
            "config": {"workload": wl.name, "cout": li.spec.cout, "cin": li.spec.cin, "tokens": li.spec.tokens,
                       "block": wl.block, "nm": f"{wl.n}:{wl.m}", "tau": wl.tau, "iters": wl.iters,
                       "parallelism": f"layer-sharded x{world}" if world > 1 else "single GPU",
                       "l2": "flushed between timed steps (256 MiB write)",
                       "path": "simt" if args.simt else "tcgen05",
                       "launch": "cuda-graph replay per step" if graph_mode else "eager launches",
                       "pdl": os.environ.get("LCP_PDL", "1") != "0"},
            "roofline": roof, "stages": per_stage, "clocks": clocks, "e2e": e2e, "e2e_all_inputs": e2e_all,
            "eager": eager,
            "gpu_launches": step.launches * K}
    if world == 1 and not args.no_extras and not args.simt:
        line["extras"] = extras(args, b, synth, wl, li, layer, step, flush, pk, dev)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
        if not args.no_extras:
            one = cpu_baseline_one_core(wl)
            if one:
                line["cpu_baseline_one_core"] = one
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def extras(args, b, synth, wl, li, layer, step, flush, pk, dev):
    """Secondary measurements of the same build, rank 0 at N = 1 only.

    - cached_dense: the step with LCP_FLAG_CACHED_DENSE (Y_d read from layer.Yd,
      written once by an uncached step), same timing protocol as the headline;
    - hard_step: the step with LCP_FLAG_HARD, and the hardening kernel alone;
    - score_step: the step with LCP_FLAG_SCORE and Wanda scores;
    - train: steps of lcp_train (step + AdamW on L, temperature schedule);
    - cublas_same_products: the two dense products of the step through torch.mm
      on the same shapes (context for the calib_gemm and bwd_gemm stages);
    - nm_mask: the standalone mask kernel on a bf16 W' of the layer's shape,
      against the measured HBM copy bandwidth (bytes: 2 read + 1/8 written per element),
      and on a 16384 x 16384 W' (nm_mask_large: its steady state);
    - sinkhorn_scaling: Sinkhorn forward then reverse over the logits of every
      projection of a 40-layer 13B-shaped model (4 x 5120^2, 2 x 13824 x 5120,
      5120 x 13824 per layer; 27 840 blocks of 64 x 64, 456 MB of float32 L) in one
      launch each, against the HBM copy bandwidth;
    - stream_ref: a plain device copy (torch) of a bf16 tensor of the layer's
      weight shape (C_out x C_in read and written: about the bytes the permute
      and block-backward stages move), L2 flushed before each, and of a ten
      times larger tensor: what a streaming kernel of that size reaches, the
      practical ceiling for the memory-bound stages.
    """
    import torch
    out = {}
    K = max(5, min(args.steps, 20))

    def want(name):
        return args.only_extra is None or args.only_extra == name

    def timed(fn, reps, flush_between=True):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        for k in range(reps):
            if flush_between:
                flush.zero_()
            e0[k].record()
            fn()
            e1[k].record()
        torch.cuda.synchronize()
        return sum(e0[k].elapsed_time(e1[k]) for k in range(reps)) / reps

    if want("cached_dense"):
        # cached dense output
        layer["Yd"] = torch.empty(li.spec.tokens, li.spec.cout, dtype=torch.float32, device=dev)
        fill = b.Step([layer], wl.block, wl.n, wl.m, wl.iters, wl.tau, workspace=step.ws)
        fill.run()
        cached = b.Step([layer], wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=b.FLAG_CACHED_DENSE, workspace=step.ws)
        g = b.capture(cached)
        ms = timed(g.replay, K)
        del g
        layer.pop("Yd")
        flop = 2 * 2 * li.spec.tokens * li.spec.cout * li.spec.cin - 2 * li.spec.tokens * li.spec.cout * li.spec.cin
        out["cached_dense"] = {"value": 1e3 / ms, "unit": UNIT, "ms_per_step": ms, "steps": K,
                               "note": "LCP_FLAG_CACHED_DENSE: Y_d = X W^T read from layer.Yd (computed once), "
                                       "so the step runs one calibration GEMM problem instead of two; "
                                       "not the headline", "algorithmic_flop": 2 * flop}

    if want("hard_step"):
        # hardened step (LCP_FLAG_HARD: per-block assignment, straight-through backward)
        nb = li.spec.cin // wl.block
        layer["perm"] = torch.empty(nb, wl.block, dtype=torch.int32, device=dev)
        hard = b.Step([layer], wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=b.FLAG_HARD)
        g = b.capture(hard)
        ms = timed(g.replay, K)
        del g
        ms_h = timed(lambda: b.harden(layer["P"], layer["perm"]), K)
        layer.pop("perm")
        # the large blocks (auction solver) on the 4096 x 4096 sweep layer's initial P
        large = {}
        for Bl in (128, 256):
            wl_l = synth.sweep_4096(Bl, 5, 1.0, 2, 4)
            Ll = torch.from_numpy(synth.make_inputs(wl_l)[0].L).to(dev)
            Pl = torch.empty_like(Ll)
            b.sinkhorn_fwd(Ll, Pl, None, wl_l.tau, wl_l.iters)
            perm_l = torch.empty(Ll.shape[0], Bl, dtype=torch.int32, device=dev)
            large[f"B{Bl}"] = {"harden_kernel_ms": timed(lambda: b.harden(Pl, perm_l), min(K, 20)),
                               "blocks": int(Ll.shape[0]), "tau": wl_l.tau}
        out["hard_step"] = {"value": 1e3 / ms, "unit": UNIT, "ms_per_step": ms, "steps": K,
                            "harden_kernel_ms": ms_h, "blocks": nb, "large_blocks": large,
                            "note": "LCP_FLAG_HARD: the forward pass uses the per-block maximum-weight "
                                    "assignment of the Sinkhorn output (B <= 64: shortest augmenting paths, "
                                    "one warp per block; B = 128, 256: epsilon-scaling auction, one CTA per "
                                    "block), the backward pass is straight-through; not the headline"}

    if want("score_step"):
        # mask from Wanda scores (LCP_FLAG_SCORE): S computed once, S_hat = S P_B ranked each step
        layer["S"] = b.score(layer["W"], layer["X"], b.SCORE_WANDA)
        sc = b.Step([layer], wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=b.FLAG_SCORE, workspace=step.ws)
        g = b.capture(sc)
        ms = timed(g.replay, K)
        del g
        layer.pop("S")
        out["score_step"] = {"value": 1e3 / ms, "unit": UNIT, "ms_per_step": ms, "steps": K, "score": "wanda",
                             "note": "LCP_FLAG_SCORE: the mask ranks S_hat = S P_B (one permute pass over S for "
                                     "the mask, one over W with that mask); not the headline"}

    if want("train"):
        # training steps: lcp_step at the scheduled temperature + AdamW on L (lcp_train)
        tr_step = b.Step([layer], wl.block, wl.n, wl.m, wl.iters, wl.tau, workspace=step.ws)
        total = 10
        trainer = b.Trainer(tr_step, b.adamw_params(lr=5e-3), total)
        ms_tr = timed(lambda: trainer.run(0, total), 3) / total
        out["train"] = {"value": 1e3 / ms_tr, "unit": UNIT, "ms_per_step": ms_tr, "steps_per_call": total,
                        "note": "lcp_train: ten steps per call (eager launches), temperature 1 -> 0.1, AdamW "
                                "lr 5e-3 on the logits after every step; L2 flushed before each call only"}

    if want("cublas_same_products"):
        # the step's two dense products through cuBLAS (torch.mm), same shapes and L2 flush, for
        # context beside the calib_gemm / bwd_gemm stages: Y_d = X W^T and Y_s = X At^T
        # (float32 outputs where torch.mm takes out_dtype, else bf16), and dAt = G^T X
        T_, co, ci = li.spec.tokens, li.spec.cout, li.spec.cin
        Xb = layer["X"] if layer["X"].dtype == torch.bfloat16 else layer["X"].to(torch.bfloat16)
        Wb = layer["W"] if layer["W"].dtype == torch.bfloat16 else layer["W"].to(torch.bfloat16)
        Gb = torch.randn(T_, co, device=dev).to(torch.bfloat16)
        try:
            torch.mm(Xb[:8], Wb[:8].t(), out_dtype=torch.float32)
            f32_out = True
        except Exception:
            f32_out = False
        kw = {"out_dtype": torch.float32} if f32_out else {}
        ms_c = timed(lambda: (torch.mm(Xb, Wb.t(), **kw), torch.mm(Xb, Wb.t(), **kw)), K)
        ms_g = timed(lambda: torch.mm(Gb.t(), Xb), K)
        fl = 2.0 * T_ * co * ci
        out["cublas_same_products"] = {
            "calib_ms": ms_c, "calib_TFLOP/s": 2 * fl / (ms_c / 1e3) / 1e12, "calib_out": "f32" if f32_out else "bf16",
            "bwd_ms": ms_g, "bwd_TFLOP/s": fl / (ms_g / 1e3) / 1e12,
            "note": "library GEMMs on the same shapes for context; the step itself runs only this build's kernels"}
        del Gb

    if want("configs"):
        # the other workload configurations (7B MLP, 13B block, the 4096^2 sweep)
        out["configs"] = config_runs(b, synth, pk, dev, flush, K)

    if want("inference_24"):
        # inference side: the layer deployed as a 2:4 compressed weight (the hard
        # permutation and mask of one LCP_FLAG_HARD step), decode-sized token counts
        out["inference_24"] = inference_24(b, layer, wl, li, dev, pk, timed, K)

    if want("nm_mask"):
        # standalone N:M mask on a bf16 W' of the layer's shape
        Wp = torch.randn(li.spec.cout, li.spec.cin, device=dev).to(torch.bfloat16)
        bits = torch.empty(li.spec.cout, li.spec.cin // 32, dtype=torch.int32, device=dev)
        ms = timed(lambda: b.nm_mask(Wp, bits, wl.n, wl.m), K)
        by = li.spec.cout * li.spec.cin * 2 + li.spec.cout * li.spec.cin // 8
        out["nm_mask"] = {"ms": ms, "GB/s": by / (ms / 1e3) / 1e9, "frac": by / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
                          "bytes": by, "shape": [li.spec.cout, li.spec.cin], "nm": f"{wl.n}:{wl.m}"}
        del Wp, bits
        # the same kernel on a 16384 x 16384 bf16 W' (512 MiB read): its steady-state bandwidth
        big = (16384, 16384)
        Wp = torch.empty(big, device=dev, dtype=torch.bfloat16).normal_()
        bits = torch.empty(big[0], big[1] // 32, dtype=torch.int32, device=dev)
        ms = timed(lambda: b.nm_mask(Wp, bits, wl.n, wl.m), K, flush_between=False)
        by = big[0] * big[1] * 2 + big[0] * big[1] // 8
        out["nm_mask_large"] = {"ms": ms, "GB/s": by / (ms / 1e3) / 1e9, "frac": by / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
                                "bytes": by, "shape": list(big), "nm": f"{wl.n}:{wl.m}",
                                "note": "input larger than L2; no flush needed"}
        del Wp, bits

    if want("stream_ref"):
        # plain copies of the layer's weight bytes and of ten times as many
        res = {}
        for name, rows, fl in (("layer", li.spec.cout, True), ("x10", li.spec.cout * 10, False)):
            src = torch.empty(rows, li.spec.cin, device=dev, dtype=torch.bfloat16).normal_()
            dst = torch.empty_like(src)
            ms = timed(lambda: dst.copy_(src), K, flush_between=fl)
            by = 2 * src.numel() * 2
            res[name] = {"ms": ms, "GB/s": by / (ms / 1e3) / 1e9, "frac": by / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
                         "bytes": by, "shape": [rows, li.spec.cin], "l2": "flushed" if fl else "larger than L2"}
            del src, dst
        out["stream_ref"] = res

    if want("sinkhorn_scaling"):
        # Sinkhorn scaling run: every projection of a 40-layer 13B-shaped model
        nblk = args.scaling_blocks
        Bk = 64
        gen = torch.Generator(device=dev).manual_seed(7)
        Lb = torch.randn(nblk, Bk, Bk, device=dev, generator=gen) * 1e-3
        Pb = torch.empty_like(Lb)
        ck = torch.empty(nblk, wl.iters, 2, Bk, device=dev)
        dP = torch.randn(nblk, Bk, Bk, device=dev, generator=gen)
        dLb = torch.empty_like(Lb)
        ms_f = timed(lambda: b.sinkhorn_fwd(Lb, Pb, ck, wl.tau, wl.iters), 5, flush_between=False)
        ms_b = timed(lambda: b.sinkhorn_bwd(Lb, ck, dP, dLb, wl.tau, wl.iters), 5, flush_between=False)
        bf = nblk * Bk * Bk * 8 + nblk * wl.iters * 2 * Bk * 4
        bb = nblk * Bk * Bk * 12 + nblk * wl.iters * 2 * Bk * 4
        out["sinkhorn_scaling"] = {
            "blocks": nblk, "B": Bk, "iters": wl.iters, "L_MB": nblk * Bk * Bk * 4 / 1e6,
            "fwd": {"ms": ms_f, "GB/s": bf / (ms_f / 1e3) / 1e9, "frac": bf / (ms_f / 1e3) / 1e9 / pk["hbm_gbs"]},
            "bwd": {"ms": ms_b, "GB/s": bb / (ms_b / 1e3) / 1e9, "frac": bb / (ms_b / 1e3) / 1e9 / pk["hbm_gbs"]},
            "note": f"inputs larger than L2 ({nblk * Bk * Bk * 4 / 1e6:.0f} MB of logits per launch)"}
        del Lb, Pb, ck, dP, dLb
        torch.cuda.empty_cache()
    return out


def config_runs(b, synth, pk, dev, flush, K):
    """The other workload configurations, each step one lcp_step call over all
    of its layers, timed like the headline (CUDA-graph replays, L2 flushed
    before each, inputs already on the device):

    - mlp_7b: gate/up 11008 x 4096 (sharing X) and down 4096 x 11008 with a
      ReLU-like input, T = 2048;
    - block_13b: the seven projections of a 13B layer (q/k/v/o 5120^2, gate/up
      13824 x 5120, down 5120 x 13824), T = 4096;
    - sweep_4096: the 32 points B x iters x tau x N:M on W 4096 x 4096, T = 2048.

    mlp_7b and block_13b also report the stage times summed over their layers
    (stage events of every layer, a separate graph) and the calibration GEMM's
    fraction of the bf16 peak."""
    import torch

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        for k in range(reps):
            flush.zero_()
            e0[k].record()
            fn()
            e1[k].record()
        torch.cuda.synchronize()
        return sum(e0[k].elapsed_time(e1[k]) for k in range(reps)) / reps

    def device_layers(inputs):
        xs, layers = {}, []
        for li in inputs:
            X = xs.get(li.spec.x_key)
            if X is None:
                X = xs[li.spec.x_key] = torch.from_numpy(li.X).to(dev).to(torch.bfloat16)
            layers.append(b.alloc_outputs(torch.from_numpy(li.W).to(dev).to(torch.bfloat16), X,
                                          torch.from_numpy(li.L).to(dev)))
        return layers

    def flops(inputs, wl):
        calib = sum(4.0 * li.spec.tokens * li.spec.cout * li.spec.cin for li in inputs)
        step = sum(6.0 * li.spec.tokens * li.spec.cout * li.spec.cin
                   + 10.0 * li.spec.cout * li.spec.cin * wl.block for li in inputs)
        return calib, step

    out = {}
    for wl in (synth.mlp_7b(), synth.block_13b()):
        inputs = synth.make_inputs(wl)
        layers = device_layers(inputs)
        st = b.Step(layers, wl.block, wl.n, wl.m, wl.iters, wl.tau)
        g = b.capture(st)
        ms = timed(g.replay, K)
        del g
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(b.TIMED_EVENTS * len(layers))]
        for e in ev:
            e.record()
        g = b.capture(st, ev)
        for _ in range(3):
            g.replay()
        reps = max(3, K // 2)
        stages = {name: 0.0 for name in b.STAGES}
        for _ in range(reps):
            flush.zero_()
            g.replay()
            torch.cuda.synchronize()
            for i in range(len(layers)):
                for k, name in enumerate(b.STAGES):
                    stages[name] += ev[b.TIMED_EVENTS * i + k].elapsed_time(ev[b.TIMED_EVENTS * i + k + 1]) / reps
        del g
        calib, total = flops(inputs, wl)
        tf = calib / (stages["calib_gemm"] / 1e3) / 1e12
        out[wl.name] = {
            "value": 1e3 / ms, "unit": "steps/s", "ms_per_step": ms, "steps": K, "layers": len(layers),
            "shapes": [[li.spec.cout, li.spec.cin, li.spec.tokens] for li in inputs],
            "launches": st.launches, "step_TFLOP/s": total / (ms / 1e3) / 1e12,
            "step_frac_bf16": total / (ms / 1e3) / 1e12 / pk["bf16_tflops"],
            "stages_ms_summed_over_layers": stages,
            "roofline_calib_gemm": {"bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                                    "frac": tf / pk["bf16_tflops"]},
            "note": "one lcp_step call over every layer per step; stage events of every layer in a second graph"}
        del st, layers, inputs
        torch.cuda.empty_cache()

    points = {}
    for B in (32, 64, 128, 256):
        inputs = synth.make_inputs(synth.sweep_4096(B, 5, 1.0, 2, 4))
        layers = device_layers(inputs)
        calib, total = flops(inputs, synth.sweep_4096(B, 5, 1.0, 2, 4))
        for it in (5, 20):
            for tau in (1.0, 0.1):
                for (n, m) in ((2, 4), (4, 8)):
                    st = b.Step(layers, B, n, m, it, tau)
                    g = b.capture(st)
                    ms = timed(g.replay, max(5, K // 2))
                    del g, st
                    points[f"B{B}_it{it}_tau{tau:g}_{n}of{m}"] = {
                        "steps/s": 1e3 / ms, "ms": ms, "step_TFLOP/s": total / (ms / 1e3) / 1e12}
        del layers, inputs
        torch.cuda.empty_cache()
    out["sweep_4096"] = {"points": points, "shape": [4096, 4096, 2048],
                         "note": "every point runs only tensor-core contractions; at B = 256 four CTAs "
                                 "share a block in the block backward, each owning a 128 x 128 quadrant of dP"}
    return out


def inference_24(b, layer, wl, li, dev, pk, timed, K):
    """The deployed layer: lcp_sparse24_mm (gather fused) against the dense
    bf16 product through cuBLAS (torch.mm) at decode-sized T, and the
    standalone gather against PyTorch's column indexing at T = 2048.

    These calls take microseconds, less than the host's cost of issuing them,
    so each is timed inside a CUDA graph of R repetitions of (L2 flush, call)
    minus a graph of R flushes alone."""
    import torch
    cout, cin, B = li.spec.cout, li.spec.cin, wl.block
    nb = cin // B
    layer["perm"] = torch.empty(nb, B, dtype=torch.int32, device=dev)
    hard = b.Step([layer], B, wl.n, wl.m, wl.iters, wl.tau, flags=b.FLAG_HARD)
    hard.run()
    perm = layer.pop("perm")
    W = layer["W"] if layer["W"].dtype == torch.bfloat16 else layer["W"].to(torch.bfloat16)
    vals, meta = b.pack24(W, perm, layer["mask"], B)
    torch.cuda.synchronize()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    R = max(5, min(K, 20))

    def graph_us(fn):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for _ in range(2):
                flush.zero_()
                if fn is not None:
                    fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(R):
                flush.zero_()
                if fn is not None:
                    fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(5):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / 5 / R * 1e3

    t_flush = graph_us(None)
    res = {"shape": [cout, cin], "B": B, "per_T": {}, "timing": f"CUDA graph of {R} x (L2 flush, call) "
                                                                 f"minus {R} flushes alone"}
    gen = torch.Generator(device=dev).manual_seed(11)
    for T in (1, 4, 8, 16):
        X = torch.randn(T, cin, device=dev, generator=gen).to(torch.bfloat16)
        Y = torch.empty(T, cout, dtype=torch.float32, device=dev)
        us_s = graph_us(lambda: b.sparse24_mm(vals, meta, X, perm, B, Y)) - t_flush
        us_d = graph_us(lambda: torch.mm(X, W.t())) - t_flush
        by = cout * cin // 2 * 2 + cout * cin // 8 + T * cin * 2 + T * cout * 4
        res["per_T"][str(T)] = {"sparse_us": us_s, "dense_cublas_us": us_d, "speedup": us_d / us_s,
                                "sparse_GB/s": by / us_s / 1e3, "sparse_frac_hbm": by / us_s / 1e3 / pk["hbm_gbs"],
                                "bytes": by}
    # the run-time permutation alone on a prefill-sized activation
    T = li.spec.tokens
    X = torch.randn(T, cin, device=dev, generator=gen).to(torch.bfloat16)
    Xp = torch.empty_like(X)
    src = torch.empty(cin, dtype=torch.long, device=dev)
    pl = perm.long()
    base = (torch.arange(nb, device=dev) * B)[:, None]
    src[(base + pl).reshape(-1)] = (base + torch.arange(B, device=dev)[None, :]).reshape(-1)
    us_g = graph_us(lambda: b.gather(X, perm, Xp)) - t_flush
    us_t = graph_us(lambda: X[:, src]) - t_flush
    assert torch.equal(X[:, src], b.gather(X, perm))
    byg = 2 * T * cin * 2
    res["gather"] = {"T": T, "us": us_g, "torch_index_us": us_t, "speedup_vs_torch": us_t / us_g,
                     "GB/s": byg / us_g / 1e3, "frac_hbm": byg / us_g / 1e3 / pk["hbm_gbs"]}
    res["note"] = ("permutation and mask from one LCP_FLAG_HARD step of the layer; bytes of the sparse "
                   "product = kept values + 4-bit position fields + X + Y")
    del flush
    return res


def cpu_baseline_one_core(wl):
    """The oracle on one BLAS thread: one whole step of the same layer."""
    from oracle import lcp_oracle as O
    from learnable_channel_permutation_b200 import synth
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        return None
    li = synth.make_inputs(wl)[0]
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        O.step(li.W, li.X, li.L, wl.tau, wl.iters, wl.n, wl.m)
        el = time.perf_counter() - t0
    return {"value": 1.0 / el, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"1 whole fwd+bwd step of the {wl.name} layer (float64 numpy oracle, one BLAS thread), "
                      f"{el:.1f} s"}


def traffic_for(kernel, simt):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if simt or not os.path.exists(p):
        return None
    d = json.load(open(p))
    ent = d.get(kernel)
    if not ent:
        return None
    try:
        if ent.get("src_hash") != src_hash(ent["sources"]):
            return None
    except OSError:
        return None
    return ent.get("bytes_per_launch")


if __name__ == "__main__":
    sys.exit(main())

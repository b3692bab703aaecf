"""The reference arm of bench.py (the oracle timed on the host cores) runs
without a GPU and prints one JSON line with the contract's keys."""
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    t0 = time.perf_counter()
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "1", "--workload", "toy_256"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    wall = time.perf_counter() - t0
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert abs(d["ms_per_step"] - 1e3 / d["value"]) <= 1e-6 * d["ms_per_step"]
    assert d["config"]["workload"] == "toy_256"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # the arm times what it prints: its K timed steps fit inside the process's wall time
    assert d["ms_per_step"] * d["steps"] / 1e3 <= wall


def test_bench_workloads_are_the_named_layers():
    """--workload names the layer it runs: the q_proj-shaped headline layer and the sweep's
    4096 x 4096 layer at B = 128 / 256 (5 iterations, tau 1.0, 2:4)."""
    sys.path.insert(0, ROOT)
    import bench
    from learnable_channel_permutation_b200 import synth
    q = bench.workload("q_proj_4096")
    assert (q.block, q.n, q.m, q.iters, q.tau) == (64, 2, 4, 5, 0.5)
    assert (q.layers[0].cout, q.layers[0].cin, q.layers[0].tokens) == (4096, 4096, 2048)
    for B in (128, 256):
        w = bench.workload(f"sweep_4096_b{B}")
        ref = synth.sweep_4096(B, 5, 1.0, 2, 4)
        assert w.name == ref.name and (w.block, w.n, w.m, w.iters, w.tau) == (B, 2, 4, 5, 1.0)
        assert [(l.cout, l.cin, l.tokens) for l in w.layers] == [(4096, 4096, 2048)]

"""Multi-process host logic of the layer-sharded benchmark, on CPU with gloo (world size 2)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from learnable_channel_permutation_b200 import parallel, synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = parallel.rank_workload(synth.custom(16, 64, 8, 32, 2, 4, 0.5, 5, "bf16", seed=0), rank)
        li = synth.make_inputs(wl)[0]
        # each rank: its own layer (distinct draws), identical shapes
        fingerprint = float(li.W.astype("float64").sum())
        got = parallel.max_over_ranks([10.0 + rank, -float(rank), fingerprint])
        q.put((rank, wl.seed, li.W.shape, got, fingerprint, parallel.shard(list(range(7)), rank, world)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_layers_and_reduce_times_with_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, sh0, got0, f0, l0), (r1, s1, sh1, got1, f1, l1) = res
    assert (s0, s1) == (0, 1) and sh0 == sh1
    assert f0 != f1                                   # independent layers
    assert got0 == got1 == [11.0, 0.0, max(f0, f1)]   # max over ranks, identical on both
    assert sorted(l0 + l1) == list(range(7)) and not set(l0) & set(l1)


def test_job_throughput_counts_every_rank():
    assert parallel.job_throughput(10, 4, 2000.0) == pytest.approx(20.0)
    assert parallel.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]   # no process group: identity


# ------------------------------------------------------- token-parallel split --

def _tp_worker(rank, world, port, T, q):
    import numpy as np
    import torch
    from oracle import lcp_oracle as O
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(7)
        W = rng.standard_normal((20, 32)) * 0.02
        X = rng.standard_normal((T, 32))
        L = rng.standard_normal((4, 8, 8)) * 0.3
        tau, iters, n, m = 0.5, 5, 2, 4
        sl = parallel.token_shard(T, rank, world)
        dP = [torch.zeros(4, 8, 8, dtype=torch.float64)]
        losses = [torch.zeros(1, dtype=torch.float64)]
        state = {}

        def run_shard():
            # the oracle stands in for lcp_step_shard: shard gradients under the global token mean
            fw = O.forward(W, X[sl], L, tau, iters, n, m)
            bw = O.backward(fw, tau)
            scale = (sl.stop - sl.start) / T
            dP[0].copy_(torch.from_numpy(bw["dP"] * scale))
            losses[0].fill_(fw["loss"] * scale)
            state["trace"], state["P"] = fw["trace"], fw["P"]

        def finish():
            state["dL"] = O.sinkhorn_backward(state["trace"], state["P"], dP[0].numpy(), tau)

        parallel.token_parallel_step(run_shard, finish, dP, losses)
        q.put((rank, sl.start, sl.stop, float(losses[0]), state["dL"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T", [30, 31])
def test_two_token_shards_all_reduce_to_the_full_batch_gradient(T):
    import numpy as np
    from oracle import lcp_oracle as O
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_tp_worker, args=(r, world, port, T, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, a0, b0, l0, d0), (_, a1, b1, l1, d1) = res
    assert (a0, b0, a1, b1) == (0, (T + 1) // 2, (T + 1) // 2, T)
    rng = np.random.default_rng(7)
    W = rng.standard_normal((20, 32)) * 0.02
    X = rng.standard_normal((T, 32))
    L = rng.standard_normal((4, 8, 8)) * 0.3
    full = O.step(W, X, L, 0.5, 5, 2, 4)
    assert l0 == l1 and abs(l0 - full["loss"]) <= 1e-14
    assert np.array_equal(d0, d1)                     # every rank holds the same whole-batch dL
    assert np.allclose(d0, full["dL"], rtol=1e-10, atol=1e-16)


def test_token_shards_cover_every_token_once():
    for world in range(1, 6):
        for T in (world, world + 1, 17, 2048):
            sl = [parallel.token_shard(T, r, world) for r in range(world)]
            assert sl[0].start == 0 and sl[-1].stop == T
            assert all(sl[r].stop == sl[r + 1].start for r in range(world - 1))
            sizes = [s.stop - s.start for s in sl]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_allreduce_without_a_process_group_is_the_identity():
    import torch
    t = [torch.arange(4.0), torch.ones(1)]
    assert parallel.allreduce_sum_(t) is t and t[0].tolist() == [0.0, 1.0, 2.0, 3.0]

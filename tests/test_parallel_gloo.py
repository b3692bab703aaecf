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

"""Multi-process host logic of the replicas mode on CPU: two gloo ranks.

Each rank of `bench.py --gpus N` trains its own replica; the job time is the
slowest rank's and the throughput counts every rank's tokens. The collective
and the arithmetic are exercised here with world size 2 on the gloo backend.
"""
import multiprocessing as mp
import socket

import numpy as np

from gpt_step_b200 import replicas, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import os
    import torch.distributed as dist
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        r, w, lr = replicas.rank_env()
        ms = 100.0 + 25.0 * rank                      # rank 1 is the slow one
        t_max = replicas.max_over_ranks(ms)
        value = replicas.job_throughput(1000, w, t_max)
        src = synth.TokenSource(2, 32, 500, replicas.replica_seed(1337, r), 40, 2)
        x, _ = src.get()
        q.put((r, w, lr, t_max, value, x.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_slowest_time_and_count_all_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for r, (rank, world, local, t_max, value, _) in enumerate(out):
        assert (rank, world, local) == (r, 2, r)
        assert t_max == 125.0                          # max over ranks, on every rank
        assert value == 1000 * 2 / 0.125               # all ranks' tokens / slowest time
    # each replica reads its own token stream
    assert not np.array_equal(np.array(out[0][5]), np.array(out[1][5]))


def test_single_process_needs_no_group():
    assert replicas.max_over_ranks(42.0) == 42.0
    assert replicas.job_throughput(500, 1, 250.0) == 2000.0

"""The replica (multi-GPU) host logic on CPU: two gloo ranks exercise the
barrier, the max-over-ranks timing and the per-rank seeds that bench.py uses
with NCCL on GPUs.  No GPU is touched."""

import os
import socket

import torch
import torch.multiprocessing as mp

from few_step_dit_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, lr = replicas.env()
    assert (r, w, lr) == (rank, world, rank)
    replicas.init(w, backend="gloo", timeout_s=60)
    dev = torch.device("cpu")
    replicas.barrier(w, dev)
    t = replicas.max_over_ranks(1.5 + rank, w, dev)
    seed = replicas.input_seed(1234, rank)
    replicas.barrier(w, dev)
    replicas.shutdown(w)
    out[rank] = (t, seed)


def test_two_gloo_ranks_agree_on_slowest_time_and_use_distinct_seeds():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 2.5
    assert out[0][1] != out[1][1]


def test_weak_scaling_value_uses_slowest_rank():
    # 2 ranks x 12,560 tokens x 3 evals, slowest rank 0.8 s
    assert replicas.weak_scaling_value(12560 * 3, 2, 0.8) == 2 * 12560 * 3 / 0.8
    assert replicas.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0

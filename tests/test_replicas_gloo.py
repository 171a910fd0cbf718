"""The multi-GPU bench path on the CPU: two gloo ranks run the same plumbing
the GPU ranks run over NCCL (barrier, max over ranks, whole-job rate, per-rank
seeds), with no GPU involved."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_112_b200 import replicas
from gated_delta_rule_112_b200.inputs import make_chunk_inputs


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r = replicas.world_and_rank()
        replicas.barrier()
        # each rank "measures" a different time; the job takes the slowest
        ms_local = 10.0 + 5.0 * r
        ms = replicas.max_over_ranks(ms_local)
        rate = replicas.job_rate(1000.0, ms, w)
        # shards are distinct sequences: different seeds, different data
        seed = replicas.shard_seed(1, r)
        inp = make_chunk_inputs("tiny_fp32", seed=seed)
        first = float(inp["q"].flatten()[0])
        gathered = [None] * w
        dist.all_gather_object(gathered, (r, seed, first))
        out[r] = (w, ms, rate, gathered)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_like_the_gpu_bench():
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        w, ms, rate, gathered = out[r]
        assert w == world
        assert ms == pytest.approx(15.0)                       # max over ranks
        assert rate == pytest.approx(world * 1000.0 / 15e-3)   # all ranks' units / slowest time
        seeds = sorted(g[1] for g in gathered)
        assert seeds == [1, 2]
        firsts = {g[1]: g[2] for g in gathered}
        assert firsts[1] != firsts[2]                         # disjoint shards


def test_single_process_makes_no_collective():
    assert not dist.is_initialized()
    assert replicas.world_and_rank() == (1, 0)
    replicas.barrier()
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.job_rate(2.0, 1.0, 1) == pytest.approx(2000.0)
    with pytest.raises(ValueError):
        replicas.job_rate(1.0, 0.0, 1)

"""The multi-rank partition of one chunked forward call, on the CPU: two gloo
ranks each run the fp64 oracle on their own shard of one input (by heads, by
equal-length sequences, by packed sequences balanced by token count), gather
the pieces, and must reproduce the unsharded oracle bit for bit (each
(sequence, head) recurrence is independent of all others)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_112_b200 import partition
from gated_delta_rule_112_b200.inputs import Workload, make_chunk_inputs

W = Workload("part", B=3, T=150, H=5, d_k=32, d_v=24, dtype=torch.float32, seed=61,
             random_state=True)
CASES = {
    "heads": dict(kw={}, by="heads"),
    "batch": dict(kw={}, by="sequences"),
    "varlen": dict(kw={"lengths": [90, 5, 0, 61, 130, 17, 44]}, by="sequences"),
}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _np(t):
    return None if t is None else t.double().numpy()


def _oracle(inp):
    import oracle
    cu = inp["cu_seqlens"]
    return oracle.chunk_fwd(_np(inp["q"]), _np(inp["k"]), _np(inp["v"]), _np(inp["g"]),
                            _np(inp["beta"]), _np(inp["initial_state"]),
                            None if cu is None else cu.numpy(), nthreads=2)


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = {}
        for name, case in CASES.items():
            inp = make_chunk_inputs(W, **case["kw"])
            parts = partition.plan(inp, world, case["by"])
            mine = partition.shard(inp, parts[rank])
            local = _oracle(mine)
            res[name] = partition.gather(inp, parts, local)
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_the_unsharded_oracle():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for name, case in CASES.items():
        ref_o, ref_fs = _oracle(make_chunk_inputs(W, **case["kw"]))
        for r in range(world):
            o, fs = out[r][name]
            assert np.array_equal(o, ref_o), (name, r)
            assert np.array_equal(fs, ref_fs), (name, r)


def test_head_ranges_cover_every_head_once():
    for H in (0, 1, 5, 16, 32):
        for world in (1, 2, 3, 8):
            rs = partition.head_ranges(H, world)
            assert len(rs) == world
            assert rs[0][0] == 0 and rs[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 1


def test_balance_sequences_is_a_balanced_partition():
    gen = torch.Generator().manual_seed(3)
    lens = [int(x) for x in torch.randint(0, 2048, (64,), generator=gen)]
    for world in (1, 2, 4, 8):
        owned = partition.balance_sequences(lens, world)
        flat = sorted(i for o in owned for i in o)
        assert flat == list(range(len(lens)))
        loads = [sum(lens[i] for i in o) for o in owned]
        # greedy longest-first: no rank exceeds the mean by more than one sequence
        assert max(loads) - sum(loads) / world <= max(lens)
    assert partition.balance_sequences([5, 5, 5, 5], 2) == [[0, 2], [1, 3]]


def test_shard_and_assemble_round_trip_on_tensors():
    inp = make_chunk_inputs(W, lengths=[30, 0, 12, 70])
    for by in ("heads", "sequences"):
        parts = partition.plan(inp, 3, by)
        outs = []
        for p in parts:
            s = partition.shard(inp, p)
            # "outputs" that are just the inputs, so the round trip is checkable
            n = s["num_seqs"] if by == "sequences" else inp["num_seqs"]
            fs = s["initial_state"] if s["initial_state"] is not None else torch.zeros(n)
            outs.append((s["v"], fs))
        o, fs = partition.assemble(inp, parts, outs)
        assert torch.equal(o, inp["v"])
        assert torch.equal(fs, inp["initial_state"])


def test_unknown_partition_is_rejected():
    with pytest.raises(ValueError):
        partition.plan(make_chunk_inputs(W), 2, "tokens")

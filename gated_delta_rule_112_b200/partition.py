"""Partition of one chunked forward call across ranks, and its reassembly.

Every (sequence, head) pair of the gated delta rule is an independent
recurrence with a fixed-size state (phantomic12 "gated-deltanet" page,
mechanism paragraph), so one call's work splits across ranks with no data
exchange on the hot path:

* by heads: rank r takes the contiguous head range ``head_ranges(H, W)[r]``
  of every sequence;
* by sequences: rank r takes a subset of the (packed) sequences, chosen by
  ``balance_sequences`` so that every rank gets about the same number of
  tokens (longest first, each to the rank with the fewest tokens so far).

``shard`` cuts a rank's inputs out of the full batch (contiguous copies, with
a rebuilt ``cu_seqlens`` for packed sequences), and ``assemble`` puts the
ranks' outputs back into the full ``o`` and ``final_state``; ``gather``
collects them over torch.distributed (any backend) and assembles them on
every rank. Only argument bookkeeping happens here: the recurrence itself runs
on each rank's shard in the library's kernels (or, in the tests, in the
oracle).
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = ["head_ranges", "balance_sequences", "plan", "shard", "assemble", "gather"]


def head_ranges(H: int, world: int) -> list[tuple[int, int]]:
    """Contiguous head ranges [h0, h1), sizes differing by at most one; with
    more ranks than heads the extra ranks get empty ranges."""
    if H < 0 or world < 1:
        raise ValueError("need H >= 0 and world >= 1")
    base, extra = divmod(H, world)
    out, h = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((h, h + n))
        h += n
    return out


def balance_sequences(lengths, world: int) -> list[list[int]]:
    """Sequence indices per rank, balanced by token count: sequences in order
    of decreasing length (ties: lower index first) each go to the rank with the
    fewest tokens so far (ties: lower rank). Each rank's list is sorted."""
    if world < 1:
        raise ValueError("world >= 1")
    lengths = [int(x) for x in lengths]
    if any(x < 0 for x in lengths):
        raise ValueError("negative sequence length")
    load = [0] * world
    owned = [[] for _ in range(world)]
    for i in sorted(range(len(lengths)), key=lambda i: (-lengths[i], i)):
        r = min(range(world), key=lambda r: (load[r], r))
        owned[r].append(i)
        load[r] += lengths[i]
    return [sorted(o) for o in owned]


def _lengths(inp) -> list[int]:
    cu = inp.get("cu_seqlens")
    if cu is None:
        return [int(inp["T"])] * int(inp["B"])
    cu = [int(x) for x in (cu.tolist() if hasattr(cu, "tolist") else cu)]
    return [cu[i + 1] - cu[i] for i in range(len(cu) - 1)]


def plan(inp, world: int, by: str = "heads") -> list[dict]:
    """One entry per rank: {"by": "heads", "h0", "h1"} or
    {"by": "sequences", "seqs": [...]} for the inputs dict ``inp`` (keys as
    returned by ``inputs.make_chunk_inputs``)."""
    if by == "heads":
        return [{"by": "heads", "h0": a, "h1": b} for a, b in head_ranges(int(inp["H"]), world)]
    if by == "sequences":
        return [{"by": "sequences", "seqs": s}
                for s in balance_sequences(_lengths(inp), world)]
    raise ValueError(f"unknown partition {by!r}")


def _cat(parts, like, dim):
    if parts:
        return torch.cat(parts, dim=dim).contiguous()
    shape = list(like.shape)
    shape[dim] = 0
    return like.new_empty(shape)


def shard(inp, part: dict) -> dict:
    """The inputs of one rank's part, as a new inputs dict (contiguous tensors
    on the device of ``inp``'s tensors)."""
    out = dict(inp)
    if part["by"] == "heads":
        h0, h1 = part["h0"], part["h1"]
        for key in ("q", "k", "v", "g", "beta"):
            out[key] = inp[key][:, :, h0:h1].contiguous()
        s0 = inp.get("initial_state")
        out["initial_state"] = None if s0 is None else s0[:, h0:h1].contiguous()
        out["H"] = h1 - h0
        return out
    seqs = part["seqs"]
    s0 = inp.get("initial_state")
    out["initial_state"] = None if s0 is None else _cat([s0[i:i + 1] for i in seqs], s0, 0)
    out["num_seqs"] = len(seqs)
    if inp.get("cu_seqlens") is None:            # equal-length batch: pick rows of B
        for key in ("q", "k", "v", "g", "beta"):
            out[key] = _cat([inp[key][i:i + 1] for i in seqs], inp[key], 0)
        out["B"] = len(seqs)
        return out
    cu = [int(x) for x in inp["cu_seqlens"].tolist()]
    for key in ("q", "k", "v", "g", "beta"):
        out[key] = _cat([inp[key][:, cu[i]:cu[i + 1]] for i in seqs], inp[key], 1)
    lens = [cu[i + 1] - cu[i] for i in seqs]
    out["cu_seqlens"] = torch.tensor([0] + list(np.cumsum(lens, dtype=np.int64)),
                                     dtype=torch.int32, device=inp["cu_seqlens"].device)
    out["T"] = int(sum(lens))
    return out


def _zeros_like_full(x, shape):
    if isinstance(x, np.ndarray):
        return np.zeros(shape, dtype=x.dtype)
    return torch.zeros(shape, dtype=x.dtype, device=x.device)


def assemble(inp, parts: list[dict], outs: list[tuple]) -> tuple:
    """Full (o, final_state) from every rank's (o, final_state), in rank order.
    Works for numpy arrays and torch tensors alike."""
    o0, f0 = outs[0]
    B, T, H = int(inp["B"]), int(inp["T"]), int(inp["H"])
    lens = _lengths(inp)
    N = len(lens)
    dv = o0.shape[-1]
    dk, dv_s = f0.shape[-2], f0.shape[-1]
    o = _zeros_like_full(o0, (B, T, H, dv))
    fs = _zeros_like_full(f0, (N, H, dk, dv_s))
    for part, (op, fp) in zip(parts, outs):
        if part["by"] == "heads":
            o[:, :, part["h0"]:part["h1"]] = op
            fs[:, part["h0"]:part["h1"]] = fp
            continue
        seqs = part["seqs"]
        if inp.get("cu_seqlens") is None:
            for j, i in enumerate(seqs):
                o[i] = op[j]
                fs[i] = fp[j]
            continue
        cu = [int(x) for x in inp["cu_seqlens"].tolist()]
        t = 0
        for j, i in enumerate(seqs):
            n = cu[i + 1] - cu[i]
            o[:, cu[i]:cu[i + 1]] = op[:, t:t + n]
            fs[i] = fp[j]
            t += n
    return o, fs


def gather(inp, parts: list[dict], local: tuple, group=None) -> tuple:
    """Collect every rank's (o, final_state) with torch.distributed and
    assemble the full result on every rank. Outside the timed hot path (it
    moves the outputs through host memory with all_gather_object)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    got = [None] * world
    as_np = tuple(x if isinstance(x, np.ndarray) else x.detach().cpu() for x in local)
    dist.all_gather_object(got, as_np, group=group)
    return assemble(inp, parts, got)

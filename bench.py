#!/usr/bin/env python
"""Benchmark of the gated delta rule hot path on B200.

One step = one chunked forward pass (gdn_chunk_fwd: chunk map, prep and scan
kernels) over the B=4, H=16, T=4096, d_k=d_v=128 bf16 workload, inputs
already resident in HBM. The decode step (N=256, H=32, d=128, fp32 state,
64 consecutive steps) is measured in the same run and reported under
"decode". Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun, one rank per GPU) the job is partitioned
with no collective on the data path (every (sequence, head) recurrence is
independent): by default every rank owns its own batch of B sequences of a
job of N*B sequences (weak scaling); ``--scaling strong`` splits the one
workload's heads across the ranks (gated_delta_rule_112_b200.partition).
Times are the max over ranks.

The long-context (long64k) and packed-varlen (varlen64) configurations are
measured in the same run and reported under their names, each against its
own algorithmic bytes. ``--impl reference`` times the CPU fp64
oracle (the slow, obviously-correct program the GPU path is checked
against) on a bounded sample of the same workload.

``--workload kda_b4h16t4096`` measures the channel-wise-gate variant instead
(gdn_kda_chunk_fwd on the tensor-core kernels, and gdn_kda_decode_step on the
kda_decode workload), against its own algorithmic bytes (g is one fp32 per
channel).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "b4h16t4096"
METRIC = "chunk-fwd Mtokens/s at B4·H16·T4096·d128 bf16; decode GB/s; % roofline"
UNIT = "Mtokens/s"
METRIC_KDA = ("chunk-fwd Mtokens/s at B4·H16·T4096·d128 bf16, channel-wise gate; "
              "decode GB/s; % roofline")
BYTES_PER_TOKEN_HEAD = 3 * 128 * 2 + 128 * 2 + 2 * 4    # q,k,v,o bf16 + g,beta fp32
BYTES_PER_TOKEN_HEAD_KDA = 3 * 128 * 2 + 128 * 2 + 128 * 4 + 4   # g is one fp32 per channel
L2_FLUSH_BYTES = 256 << 20
# Chunked-forward configurations measured beside the headline one.
EXTRA_WORKLOADS = ("long64k", "varlen64")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--decode-n", type=int, default=0,
                   help="sequences of the decode step (default: the workload's 256; a smaller "
                        "count makes a small case of the same kernel for profiler captures)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--scaling", choices=["weak", "strong"], default="weak",
                   help="N > 1: weak = every rank owns B sequences of a job of N*B "
                        "sequences; strong = one workload split by heads across the ranks")
    p.add_argument("--no-extra-workloads", action="store_true",
                   help="skip the long64k and varlen64 sub-measurements")
    p.add_argument("--bwd", action="store_true",
                   help="time the backward pass (the default; kept for older command lines)")
    p.add_argument("--no-bwd", action="store_true",
                   help="skip the backward-pass and training-step sub-measurements")
    p.add_argument("--workload", default=WORKLOAD,
                   help="chunked-forward workload (inputs.WORKLOADS); the default is the "
                        "headline configuration, the others are for extra measurements")
    return p.parse_args()


# The sources each measured kernel set is built from (under csrc/).
KERNEL_SOURCES = {
    "chunk_fwd_step": ["chunk_map.cu", "chunk_tc.cu", "gdn_internal.cuh", "sm100_ptx.cuh"],
    "kda_chunk_fwd_step": ["chunk_map.cu", "chunk_tc.cu", "gdn_internal.cuh", "sm100_ptx.cuh"],
    "decode": ["decode.cu", "gdn_internal.cuh", "sm100_ptx.cuh"],
    "bwd_step": ["chunk_bwd_tc.cu", "chunk_map.cu", "chunk_tc.cu", "bwd_internal.cuh",
                 "gdn_internal.cuh", "sm100_ptx.cuh"],
}


def kernel_source_hash(kind: str) -> str:
    """Hash of the sources of one kernel set: ncu traffic figures are only
    reported for the exact kernels they were measured on."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kind]:
        h.update(open(os.path.join(ROOT, "gated_delta_rule_112_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(key):
    """DRAM bytes per launch recorded for `key` ("<kind>/<workload>"), or None
    when there is no record or the kernels changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(key)
    if not rec or rec.get("src_hash") != kernel_source_hash(key.split("/")[0]):
        return None
    return rec["dram_bytes_per_launch"]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    """Time the CPU fp64 oracle on a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import oracle
    from gated_delta_rule_112_b200.inputs import make_chunk_inputs
    inp = make_chunk_inputs(args.workload)
    kda = inp["gate"] == "channel"
    run = oracle.kda_chunk_fwd if kda else oracle.chunk_fwd
    heads = [0, 1]                              # sample: 2 of 16 heads, all B*T tokens
    arr = {k: inp[k][:, :, heads].float().double().numpy() for k in ("q", "k", "v", "g", "beta")}
    cores = oracle.default_threads()
    tok_equiv = inp["B"] * inp["T"] * len(heads) / inp["H"]

    s0 = (inp["initial_state"][:, heads].double().numpy()
          if inp["initial_state"] is not None else None)
    cu = inp["cu_seqlens"].numpy() if inp["cu_seqlens"] is not None else None

    def one():
        run(arr["q"], arr["k"], arr["v"], arr["g"], arr["beta"], s0, cu, nthreads=cores)
    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    value = tok_equiv / dt / 1e6
    sample = (f"oracle on {len(heads)} of {inp['H']} heads x B{inp['B']} x T{inp['T']} "
              f"per step ({int(tok_equiv)} full-width tokens)")
    line = {"impl": "reference", "metric": METRIC_KDA if kda else METRIC, "value": value,
            "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "B": inp["B"], "T": inp["T"], "H": inp["H"],
                       "d_k": 128, "d_v": 128, "chunk": 64},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm
def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    import gated_delta_rule_112_b200 as gdn
    from gated_delta_rule_112_b200.inputs import WORKLOADS, make_chunk_inputs, make_decode_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus > 1 and world != args.gpus:
        raise SystemExit("--gpus N > 1 must be launched with torchrun --nproc-per-node N")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    from gated_delta_rule_112_b200 import partition, replicas
    strong = args.scaling == "strong" and world > 1
    if strong and world > WORKLOADS[args.workload].H:
        raise SystemExit("--scaling strong needs at least one head per rank")
    # Whole-job rate: weak scaling counts every rank's tokens, strong scaling
    # the one workload's tokens (each rank did a part of every token).
    def job_value(tokens, ms):
        return tokens / (ms * 1e-3) if strong else replicas.job_rate(tokens, ms, world)

    barrier = replicas.barrier

    def max_over_ranks(x):
        return replicas.max_over_ranks(x, dev)

    pk = peaks()
    stream = torch.cuda.current_stream()
    L = gdn.lib()

    # --------------------------------------------------------------- chunked forward
    wl = args.workload
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    K = args.steps

    def measure_chunk(wname, steps, warmup, sampler=None):
        """Time `steps` chunked forward passes of workload `wname` (inputs
        resident in HBM, L2 flushed before each step) and, in a separate untimed
        pass, the per-kernel split. Returns the tensors and the figures."""
        if strong:
            # one workload (one seed) split by heads; this rank runs its range
            inp = make_chunk_inputs(wname)
            inp = partition.shard(inp, partition.plan(inp, world, "heads")[rank])
        else:
            # weak scaling: the job is `world` batches of sequences, rank r owning
            # the r-th (drawn with its own seed); no data crosses ranks
            inp = make_chunk_inputs(wname, seed=replicas.shard_seed(WORKLOADS[wname].seed, rank))
        kda = inp["gate"] == "channel"
        fwd = gdn.kda_chunk_fwd if kda else gdn.chunk_fwd
        ws_size = gdn.kda_workspace_size if kda else gdn.workspace_size
        B, T, H = inp["B"], inp["T"], inp["H"]
        t = {x: inp[x].to(dev) for x in ("q", "k", "v", "g", "beta")}
        s0 = inp["initial_state"].to(dev) if inp["initial_state"] is not None else None
        cu = inp["cu_seqlens"].to(dev) if inp["cu_seqlens"] is not None else None
        nseq = B if cu is None else cu.numel() - 1
        o = torch.empty(B, T, H, 128, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(ws_size(B, T, H, 128, 128, 0 if cu is None else nseq),
                         dtype=torch.uint8, device=dev)

        def step():
            return fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], s0, cu, out=o, workspace=ws)

        for _ in range(max(warmup, 3)):
            step()
        torch.cuda.synchronize()
        assert gdn.get_status(ws) == gdn.OK
        # Timed region: one event pair around each step. The kernels of a step
        # start with programmatic dependent launch; an event between them would
        # serialise them, so the per-kernel split comes from a separate pass.
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for e in evs:                  # torch creates the CUDA event on first record
            for x in e:
                x.record(stream)
        if sampler is not None:
            sampler.start()
        barrier()
        torch.cuda.synchronize()
        for i in range(steps):
            flush.fill_(i & 0xFF)                       # evict L2 between timed steps
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        barrier()
        clocks = sampler.stop() if sampler is not None else None
        status = gdn.get_status(ws)
        if status != gdn.OK:
            raise SystemExit(f"device status {status}")
        ms_local = sum(a.elapsed_time(b) for a, b in evs) / steps
        ms = max_over_ranks(ms_local)
        # Per-kernel split (untimed pass): events recorded between the launches.
        kp = min(steps, 10)
        pev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(kp)]
        for e in pev:
            for x in e:
                x.record(stream)
        torch.cuda.synchronize()
        for i in range(kp):
            flush.fill_(i & 0xFF)
            e = pev[i]
            L.gdn_set_profile_events(e[0].cuda_event, e[1].cuda_event, e[2].cuda_event,
                                     e[3].cuda_event)
            step()
        L.gdn_set_profile_events(None, None, None, None)
        torch.cuda.synchronize()
        t_map = statistics.mean(e[0].elapsed_time(e[1]) for e in pev)
        t_prep = statistics.mean(e[1].elapsed_time(e[2]) for e in pev)
        t_scan = statistics.mean(e[2].elapsed_time(e[3]) for e in pev)
        tokens = B * T if cu is None else int(inp["cu_seqlens"][-1])
        state_io = (2 if s0 is not None else 1) * nseq * H * 128 * 128 * 4   # final (+ initial)
        alg_bytes = tokens * H * (BYTES_PER_TOKEN_HEAD_KDA if kda else BYTES_PER_TOKEN_HEAD) \
            + state_io
        flops = tokens * H * 2 * (3 * 64 * 128 + 2 * 64 * 128 + 3 * 128 * 128)
        kernels = {"gdn_chunk_map_kernel": t_map,
                   ("gdn_kda_prep_kernel" if kda else "gdn_prep_kernel"): t_prep,
                   "gdn_scan_kernel": t_scan}
        segs = int(L.gdn_chunk_fwd_scan_segments(
            B, T, H, 128, 128, 0 if cu is None else nseq, 64, gdn.BF16,
            torch.cuda.get_device_properties(dev).multi_processor_count))
        launches = 3 if segs <= 1 else 5
        return dict(inp=inp, kda=kda, fwd=fwd, t=t, s0=s0, cu=cu, o=o, ws=ws, B=B, T=T, H=H,
                    nseq=nseq, tokens=tokens, ms=ms, ms_local=ms_local, alg_bytes=alg_bytes,
                    flops=flops, kernels=kernels, clocks=clocks, launches=launches, segs=segs)

    def workload_summary(r, steps):
        gbs = r["alg_bytes"] / (r["ms_local"] * 1e-3) / 1e9
        tot = sum(r["kernels"].values())
        return {"workload": r["wname"], "tokens": r["tokens"], "heads": r["H"],
                "sequences": r["nseq"], "ms_per_step": r["ms"], "steps": steps,
                "value": job_value(r["tokens"], r["ms"]) / 1e6, "unit": UNIT,
                "gpu_launches": r["launches"] * steps, "scan_segments": r["segs"],
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                             "frac": gbs / pk["hbm"], "algorithmic_bytes": r["alg_bytes"],
                             "traffic": recorded_traffic("chunk_fwd_step/" + r["wname"]),
                             "peak_source": pk["source"]},
                "kernels_ms": r["kernels"],
                "kernel_share": {k2: v2 / tot for k2, v2 in r["kernels"].items()}}

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    main_r = measure_chunk(wl, K, args.warmup, sampler)
    main_r["wname"] = wl
    inp, kda, fwd = main_r["inp"], main_r["kda"], main_r["fwd"]
    q, k, v, g, beta = (main_r["t"][x] for x in ("q", "k", "v", "g", "beta"))
    s0, cu, o, ws = main_r["s0"], main_r["cu"], main_r["o"], main_r["ws"]
    B, T, H, nseq, tokens = main_r["B"], main_r["T"], main_r["H"], main_r["nseq"], main_r["tokens"]
    ms, ms_local, clocks = main_r["ms"], main_r["ms_local"], main_r["clocks"]
    alg_bytes, flops, kernels = main_r["alg_bytes"], main_r["flops"], main_r["kernels"]
    fs = torch.empty(nseq, H, 128, 128, dtype=torch.float32, device=dev)
    value = job_value(tokens, ms) / 1e6
    ach_gbs = alg_bytes / (ms_local * 1e-3) / 1e9
    tot = sum(kernels.values())
    traffic = recorded_traffic(("kda_chunk_fwd_step/" if kda else "chunk_fwd_step/") + wl)

    # The other chunked-forward configurations (long context; packed varlen),
    # each with its own roofline against its own algorithmic bytes.
    others = {}
    if wl == WORKLOAD and not args.no_extra_workloads:
        for extra in EXTRA_WORKLOADS:
            r = measure_chunk(extra, min(K, 10), 3)
            r["wname"] = extra
            others[extra] = workload_summary(r, min(K, 10))
            del r
            torch.cuda.empty_cache()

    # --------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hg, hb = (inp[x].pin_memory() for x in ("q", "k", "v", "g", "beta"))
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        hfs = torch.empty(fs.shape, dtype=fs.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hg, hb))
        d2h = ho.numel() * ho.element_size() + hfs.numel() * hfs.element_size()

        def e2e_step_with_state():
            for dst, src in ((q, hq), (k, hk), (v, hv), (g, hg), (beta, hb)):
                dst.copy_(src, non_blocking=True)
            _, f = fwd(q, k, v, g, beta, s0, cu, out=o, workspace=ws)
            ho.copy_(o, non_blocking=True)
            hfs.copy_(f, non_blocking=True)

        for _ in range(3):
            e2e_step_with_state()
        torch.cuda.synchronize()
        ke = max(3, min(K, 10))
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(ke)]
        barrier()
        torch.cuda.synchronize()
        for i in range(ke):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            e2e_step_with_state()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_e2e = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / ke)
        e2e = {"value": job_value(tokens, ms_e2e) / 1e6, "unit": UNIT,
               "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": ke,
               "api": ("gated_delta_rule_112_b200.kda_chunk_fwd (C ABI gdn_kda_chunk_fwd)" if kda
                       else "gated_delta_rule_112_b200.chunk_fwd (C ABI gdn_chunk_fwd)")}
        del hq, hk, hv, hg, hb, ho, hfs

    # --------------------------------------------------------------- backward pass
    backward = None
    if not args.no_bwd and not kda:
        del ws
        torch.cuda.empty_cache()
        gen = torch.Generator("cpu").manual_seed(1000 + rank)
        d_o = torch.randn(B, T, H, 128, generator=gen).to(torch.bfloat16).to(dev)
        dsN = (0.1 * torch.randn(nseq, H, 128, 128, generator=gen)).to(dev)
        bws = torch.empty(gdn.bwd_workspace_size(B, T, H, 128, 128, 0 if cu is None else nseq),
                          dtype=torch.uint8, device=dev)

        def bstep():
            return gdn.chunk_bwd(q, k, v, g, beta, d_o, s0, cu, dsN, workspace=bws)

        for _ in range(3):
            bstep()
        torch.cuda.synchronize()
        assert gdn.get_status(bws) == gdn.OK
        kb = max(1, min(K, 5))
        bev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(kb)]
        barrier()
        torch.cuda.synchronize()
        for i in range(kb):
            flush.fill_(i & 0xFF)
            bev[i][0].record(stream)
            bstep()
            bev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_b = max_over_ranks(sum(a.elapsed_time(b) for a, b in bev) / kb)
        # the operation's own bytes: q, k, v, d_o bf16 and g, beta in; dq, dk, dv fp32 and
        # dg, dbeta out; the final-state gradient in and the initial-state gradient out
        bw_bytes = tokens * H * (4 * 128 * 2 + 2 * 4 + 3 * 128 * 4 + 2 * 4) + \
            (2 + (1 if s0 is not None else 0)) * nseq * H * 128 * 128 * 4
        # per (chunk, head): the forward's intermediates written and read back (48.5 KB
        # each way), the entering state S_c and the state gradient dS_{c+1} (bf16 32 KB
        # each, written once and read by the unit kernel)
        units = -(-T // 64) * H * nseq if cu is None else (tokens // 64 + nseq) * H
        scratch = units * (2 * 49664 + 2 * 2 * 32768)
        gbs_b = bw_bytes / (ms_b * 1e-3) / 1e9
        backward = {"workload": wl, "ms_per_step": ms_b, "steps": kb, "warmup": 3,
                    "value": replicas.job_rate(tokens, ms_b, world) / 1e6, "unit": UNIT,
                    "gpu_launches": 5 * kb,
                    "api": "gated_delta_rule_112_b200.chunk_bwd (C ABI gdn_chunk_bwd)",
                    "roofline": {"bound": "hbm", "achieved": gbs_b, "peak": pk["hbm"],
                                 "unit": "GB/s", "frac": gbs_b / pk["hbm"],
                                 "algorithmic_bytes": bw_bytes,
                                 "scratch_bytes": scratch,
                                 "traffic": recorded_traffic("bwd_step/" + wl),
                                 "scratch_frac": scratch / (ms_b * 1e-3) / 1e9 / pk["hbm"],
                                 "kernel": "chunk_map + prep + scan (replay, chunk states) + "
                                           "gdn_bwd_chain_kernel + gdn_bwd_unit_kernel",
                                 "peak_source": pk["source"]}}
        # A training step: the forward keeping its intermediates and chunk states
        # (gdn_chunk_fwd_save), then the backward from them (gdn_chunk_bwd_saved,
        # no replay); and that backward alone, after one saving forward.
        o_t = torch.empty_like(v)

        def tstep():
            gdn.chunk_fwd_save(q, k, v, g, beta, s0, cu, workspace=bws, out=o_t)
            return gdn.chunk_bwd_saved(q, k, v, g, beta, d_o, bws, s0, cu, dsN)

        def timed(fn):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            assert gdn.get_status(bws) == gdn.OK
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(kb)]
            barrier()
            torch.cuda.synchronize()
            for i in range(kb):
                flush.fill_(i & 0xFF)
                ev[i][0].record(stream)
                fn()
                ev[i][1].record(stream)
            torch.cuda.synchronize()
            barrier()
            return max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / kb)

        ms_t = timed(tstep)
        gdn.chunk_fwd_save(q, k, v, g, beta, s0, cu, workspace=bws, out=o_t)
        ms_bs = timed(lambda: gdn.chunk_bwd_saved(q, k, v, g, beta, d_o, bws, s0, cu, dsN))
        backward["training_step"] = {
            "ms_per_step": ms_t, "value": replicas.job_rate(tokens, ms_t, world) / 1e6,
            "unit": UNIT, "gpu_launches": 5 * kb,
            "api": "chunk_fwd_save + chunk_bwd_saved (C ABI gdn_chunk_fwd_save, "
                   "gdn_chunk_bwd_saved)",
            "backward_saved_ms": ms_bs,
            "replaying_pair_ms": ms + ms_b,
            "note": "forward with its intermediates and chunk states kept, then the backward "
                    "from them (no replay); replaying_pair_ms = the forward step above plus "
                    "the replaying backward"}
        del d_o, dsN, bws, o_t
        ws = None

    del q, k, v, g, beta, o, ws
    torch.cuda.empty_cache()

    # --------------------------------------------------------------- decode step
    decode = None
    if not args.no_decode:
        dwl = "kda_decode" if kda else "decode"
        d = make_decode_inputs(dwl, seed=replicas.shard_seed(WORKLOADS[dwl].seed, rank),
                               N=args.decode_n or None)
        dstep = gdn.kda_decode_step if kda else gdn.decode_step
        N, Hd, S = d["N"], d["H"], d["steps"]
        dq, dk, dvv, dg, db = (d[x].to(dev) for x in ("q", "k", "v", "g", "beta"))
        st = d["state"].to(dev)
        do = torch.empty(N, Hd, 128, dtype=torch.bfloat16, device=dev)
        for t in range(3):
            dstep(dq[t], dk[t], dvv[t], dg[t], db[t], st, out=do)
        st.copy_(d["state"].to(dev))
        torch.cuda.synchronize()
        reps = 3
        times = []
        barrier()
        for r in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record(stream)
            for t in range(S):
                dstep(dq[t], dk[t], dvv[t], dg[t], db[t], st, out=do)
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b) / S)
        barrier()
        us = max_over_ranks(statistics.median(times)) * 1e3
        bytes_step = (2 * N * Hd * 128 * 128 * 4 + 3 * N * Hd * 128 * 2 + N * Hd * 128 * 2
                      + N * Hd * 4 + N * Hd * (128 if kda else 1) * 4)
        gbs = bytes_step / (us * 1e-6) / 1e9
        decode = {"workload": f"{dwl} N{N} H{Hd} d128 fp32 state, {S} steps", "us_per_step": us,
                  "value": world * gbs, "unit": "GB/s", "bytes_per_step": bytes_step,
                  "gpu_launches": reps * S,
                  "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"],
                               "unit": "GB/s", "frac": gbs / pk["hbm"],
                               "traffic": recorded_traffic(f"decode/{dwl}_n{N}h{Hd}"),
                               "kernel": "gdn_decode_kernel", "peak_source": pk["source"]}}
        del dq, dk, dvv, dg, db, st, do

    # --------------------------------------------------------------- CPU baseline (oracle)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        arr = {x: inp[x].float().double().numpy() for x in ("q", "k", "v", "g", "beta")}
        cores = oracle.default_threads()
        t0 = time.perf_counter()
        (oracle.kda_chunk_fwd if kda else oracle.chunk_fwd)(
            arr["q"], arr["k"], arr["v"], arr["g"], arr["beta"], None, None, nthreads=cores)
        dt = time.perf_counter() - t0
        cpu = {"value": tokens / dt / 1e6, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"the whole workload once (B{B} T{T} H{H}, {dt:.2f} s)"}

    roof = {"bound": "hbm", "achieved": ach_gbs, "peak": pk["hbm"], "unit": "GB/s",
            "frac": ach_gbs / pk["hbm"], "traffic": traffic,
            "kernel": ("gdn_kda_chunk_fwd step (chunk_map + kda prep + scan)" if kda
                       else "gdn_chunk_fwd step (chunk_map + prep + scan)"),
            "algorithmic_bytes": alg_bytes, "flops": flops,
            "tensor_frac": flops / (ms_local * 1e-3) / (pk["bf16"] * 1e12),
            "peak_source": pk["source"]}
    line = {
        "metric": METRIC_KDA if kda else METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong" if strong else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl, "B": B, "T": T, "H": H, "d_k": 128, "d_v": 128,
                   "chunk": 64, "sequences": nseq,
                   "gate": "channel-wise [B,T,H,d_k]" if kda else "scalar [B,T,H]",
                   "initial_state": "zeros" if s0 is None else "random",
                   "final_state": True,
                   "l2": "flushed before every timed step (256 MiB device write)",
                   "parallelism": (f"{world} ranks, heads split across ranks, no collective"
                                   if strong else f"{world} rank(s), each owning its own "
                                   f"batch of sequences, no collective")},
        "roofline": roof,
        "kernels_ms": kernels,
        "kernel_share": {k2: v2 / tot for k2, v2 in kernels.items()},
        "kernels_note": "per-kernel times from an untimed pass with events between the "
                        "launches (no launch overlap); ms_per_step is the timed region",
        "gpu_launches": main_r["launches"] * K,
        "clocks": clocks,
        "e2e": e2e,
        "decode": decode,
        "backward": backward,
        "cpu_baseline": cpu,
    }
    line.update(others)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    if len(sys.argv) == 2 and sys.argv[1] == "--source-hashes":
        print(json.dumps({kind: kernel_source_hash(kind) for kind in KERNEL_SOURCES}))
    else:
        main()

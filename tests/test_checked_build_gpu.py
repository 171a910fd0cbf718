"""The bounds-checked build (libgdn_checked.so, -DGDN_CHECKS=1): the small
tensor-core parity cases run through it in a fresh process, every call must
leave no recorded out-of-bounds index (gdn_get_status == GDN_OK) and still
match the oracle. This build is the stand-in for a memory checker: it checks
every plain global-memory index of the chunk map, prep, state-scan and
segment-composition kernels against its buffer before the access."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cases():
    import numpy as np
    import torch

    import gated_delta_rule_112_b200 as gdn
    from gated_delta_rule_112_b200.inputs import Workload, make_chunk_inputs
    from tests.parity import TOL_BF16, assert_close, np64, oracle_chunk, to_dev

    assert gdn.lib().gdn_checked_build() == 1, "not the checked library"
    w = Workload("chk", B=1, T=64, H=1, d_k=128, d_v=128, seed=71)
    cases = [
        make_chunk_inputs(w, T=1),
        make_chunk_inputs(w, B=2, H=3, T=193, random_state=True),
        make_chunk_inputs(w, H=2, lengths=[70, 0, 1, 130, 64], random_state=True),
        make_chunk_inputs(w, B=1, H=1, T=64 * 40 + 37, random_state=True),   # segmented scan
        make_chunk_inputs(w, B=2, H=2, T=0, random_state=True),
    ]
    for inp in cases:
        d = to_dev(inp)
        num_seqs = inp["num_seqs"] if inp["cu_seqlens"] is not None else 0
        ws = torch.empty(gdn.workspace_size(inp["B"], inp["T"], inp["H"], 128, 128, num_seqs),
                         dtype=torch.uint8, device="cuda")
        o, fs = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"],
                              d["cu_seqlens"], workspace=ws)
        status = gdn.get_status(ws)
        assert status == gdn.OK, gdn.lib().gdn_status_string(status)
        if inp["T"] > 0:
            ro, rfs = oracle_chunk(inp)
            assert_close("o", np64(o), ro, TOL_BF16)
            assert_close("final_state", np64(fs), rfs, TOL_BF16)
        else:
            assert np.array_equal(np64(fs), np64(inp["initial_state"]))
    # the channel-wise gate's tensor-core path (its own prep kernel)
    import oracle
    wk = Workload("chk_kda", B=1, T=64, H=1, d_k=128, d_v=128, seed=72, gate="channel")
    for inp in (make_chunk_inputs(wk, B=2, H=3, T=193, random_state=True),
                make_chunk_inputs(wk, H=2, lengths=[70, 0, 1, 130, 64], random_state=True)):
        d = to_dev(inp)
        num_seqs = inp["num_seqs"] if inp["cu_seqlens"] is not None else 0
        ws = torch.empty(gdn.kda_workspace_size(inp["B"], inp["T"], inp["H"], 128, 128, num_seqs),
                         dtype=torch.uint8, device="cuda")
        o, fs = gdn.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                  d["initial_state"], d["cu_seqlens"], workspace=ws)
        status = gdn.get_status(ws)
        assert status == gdn.OK, gdn.lib().gdn_status_string(status)
        cu = inp["cu_seqlens"]
        ro, rfs = oracle.kda_chunk_fwd(np64(inp["q"]), np64(inp["k"]), np64(inp["v"]),
                                       np64(inp["g"]), np64(inp["beta"]),
                                       np64(inp["initial_state"]),
                                       None if cu is None else cu.numpy())
        assert_close("o", np64(o), ro, TOL_BF16)
        assert_close("final_state", np64(fs), rfs, TOL_BF16)
    # the chunkwise backward (forward replay with chunk states, reverse chain,
    # per-unit gradients)
    wb = Workload("chk_bwd", B=1, T=64, H=1, d_k=128, d_v=128, seed=73)
    for inp in (make_chunk_inputs(wb, B=2, H=3, T=193, random_state=True),
                make_chunk_inputs(wb, H=2, lengths=[70, 0, 1, 130, 64], random_state=True)):
        d = to_dev(inp)
        gen = torch.Generator("cpu").manual_seed(5)
        d_o = torch.randn(inp["B"], inp["T"], inp["H"], 128, generator=gen).to(torch.bfloat16)
        dsN = 0.1 * torch.randn(inp["num_seqs"], inp["H"], 128, 128, generator=gen)
        num_seqs = inp["num_seqs"] if inp["cu_seqlens"] is not None else 0
        ws = torch.empty(gdn.bwd_workspace_size(inp["B"], inp["T"], inp["H"], 128, 128, num_seqs),
                         dtype=torch.uint8, device="cuda")
        got = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d_o.cuda(),
                            d["initial_state"], d["cu_seqlens"], dsN.cuda(), workspace=ws)
        status = gdn.get_status(ws)
        assert status == gdn.OK, gdn.lib().gdn_status_string(status)
        cu = inp["cu_seqlens"]
        ref = oracle.chunk_bwd(np64(inp["q"]), np64(inp["k"]), np64(inp["v"]), np64(inp["g"]),
                               np64(inp["beta"]), np64(d_o), np64(inp["initial_state"]),
                               None if cu is None else cu.numpy(), np64(dsN))
        for key in ("dq", "dk", "dv", "dg", "dbeta", "d_initial_state"):
            assert_close(key, np64(got[key]), ref[key], TOL_BF16)
    print("checked build: all cases clean")


@pytest.mark.gpu
def test_checked_build_runs_the_tensor_core_cases_clean():
    from gated_delta_rule_112_b200 import build as gbuild
    lib = gbuild.build(checked=True)
    env = dict(os.environ, GDN_LIBRARY=lib, PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, os.path.abspath(__file__)], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-3000:]
    assert "all cases clean" in out.stdout


if __name__ == "__main__":
    sys.path.insert(0, ROOT)
    _cases()

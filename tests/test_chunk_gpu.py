"""GPU parity of gdn_chunk_fwd (tensor-core and CUDA-core paths) against the
fp64 oracle on the same seeded inputs, through the C ABI."""
import numpy as np
import pytest
import torch

from gated_delta_rule_112_b200.inputs import Workload, make_chunk_inputs
from tests.parity import (TOL_BF16, TOL_F32, assert_close, gpu_chunk, np64, oracle_chunk,
                          rel_l2, to_dev)

pytestmark = pytest.mark.gpu

SMALL = Workload("small", B=1, T=64, H=1, d_k=128, d_v=128, seed=11)


def check(inp, tol, force_simt=False, chunk=None, heads=None):
    o, fs = gpu_chunk(inp, force_simt=force_simt, chunk=chunk)
    ro, rfs = oracle_chunk(inp, heads)
    if heads is not None:
        o, fs = o[:, :, heads], fs[:, heads]
    assert_close("o", np64(o), ro, tol)
    assert_close("final_state", np64(fs), rfs, tol)
    return o, fs


# ---------------------------------------------------------------- tensor-core path
def test_tc_path_is_selected():
    import gated_delta_rule_112_b200 as gdn
    assert gdn.chunk_path(128, 128, 64, torch.bfloat16) == gdn.PATH_TCGEN05


@pytest.mark.parametrize("T", [64, 1, 63, 65, 130, 200])
def test_tc_one_head_ragged_lengths(T):
    check(make_chunk_inputs(SMALL, T=T), TOL_BF16)


@pytest.mark.parametrize("B,H,T", [(2, 3, 256), (3, 2, 193)])
def test_tc_batch_heads_with_initial_state(B, H, T):
    check(make_chunk_inputs(SMALL, B=B, H=H, T=T, random_state=True), TOL_BF16)


def test_tc_varlen_odd_lengths_with_states():
    check(make_chunk_inputs(SMALL, H=2, lengths=[70, 1, 130, 64, 5], random_state=True),
          TOL_BF16)


def test_tc_empty_sequences_keep_their_state():
    inp = make_chunk_inputs(SMALL, H=2, lengths=[0, 40, 0, 3], random_state=True)
    o, fs = check(inp, TOL_BF16)
    s0 = inp["initial_state"]
    np.testing.assert_array_equal(np64(fs[0]), np64(s0[0]))
    np.testing.assert_array_equal(np64(fs[2]), np64(s0[2]))


def test_tc_zero_tokens():
    inp = make_chunk_inputs(SMALL, B=2, H=2, T=0, random_state=True)
    o, fs = gpu_chunk(inp)
    assert o.shape == (2, 0, 2, 128)
    np.testing.assert_array_equal(np64(fs), np64(inp["initial_state"]))


def test_tc_negative_eigenvalue_beta_up_to_two():
    inp = make_chunk_inputs(SMALL, B=2, H=2, T=256, random_state=True)
    inp["beta"] = 2.0 * inp["beta"]
    check(inp, TOL_BF16)


def test_tc_matches_simt_on_same_bf16_inputs():
    inp = make_chunk_inputs(SMALL, B=2, H=2, T=320, random_state=True)
    o1, f1 = gpu_chunk(inp)
    o2, f2 = gpu_chunk(inp, force_simt=True)
    assert rel_l2(np64(o1), np64(o2)) < TOL_BF16
    assert rel_l2(np64(f1), np64(f2)) < TOL_BF16


def test_tc_split_sequence_hands_over_state():
    inp = make_chunk_inputs(SMALL, B=2, H=2, T=320, random_state=True)
    o, fs = gpu_chunk(inp)
    a = {k: v for k, v in inp.items()}
    b = {k: v for k, v in inp.items()}
    for key in ("q", "k", "v", "g", "beta"):
        a[key] = inp[key][:, :128].contiguous()
        b[key] = inp[key][:, 128:].contiguous()
    a["T"], b["T"] = 128, 192
    oa, fa = gpu_chunk(a)
    b["initial_state"] = fa.cpu()
    ob, fb = gpu_chunk(b)
    ro, rfs = oracle_chunk(inp)
    assert_close("o (split)", np64(torch.cat([oa, ob], 1)), ro, TOL_BF16)
    assert_close("final (split)", np64(fb), rfs, TOL_BF16)


def test_tc_varlen_equals_separate_calls():
    lens = [100, 64, 37]
    inp = make_chunk_inputs(SMALL, H=2, lengths=lens, random_state=True)
    o, fs = gpu_chunk(inp)
    cu = inp["cu_seqlens"].tolist()
    for n in range(len(lens)):
        one = {k: v for k, v in inp.items()}
        for key in ("q", "k", "v", "g", "beta"):
            one[key] = inp[key][:, cu[n]:cu[n + 1]].contiguous()
        one["initial_state"] = inp["initial_state"][n:n + 1].contiguous()
        one["cu_seqlens"] = None
        one["T"] = lens[n]
        on, fn = gpu_chunk(one)
        assert rel_l2(np64(on), np64(o[:, cu[n]:cu[n + 1]])) < 1e-6
        assert rel_l2(np64(fn[0]), np64(fs[n])) < 1e-6


def test_bad_cu_seqlens_reported_by_status():
    import gated_delta_rule_112_b200 as gdn
    inp = make_chunk_inputs(SMALL, H=1, lengths=[30, 34])
    d = to_dev(inp)
    bad = torch.tensor([0, 40, 30], dtype=torch.int32, device="cuda")   # not monotone
    ws = torch.empty(gdn.workspace_size(1, 64, 1, 128, 128, 2), dtype=torch.uint8,
                     device="cuda")
    gdn.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, bad, workspace=ws)
    assert gdn.get_status(ws) == gdn.ERR_INVALID_ARG
    assert gdn.get_status(ws) == gdn.OK                                  # cleared


# ---------------------------------------------------------------- CUDA-core path
@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("dk,dv", [(64, 64), (48, 80), (128, 32)])
def test_simt_fp32_small(chunk, dk, dv):
    w = Workload("s", B=2, T=77, H=2, d_k=dk, d_v=dv, dtype=torch.float32, seed=5)
    check(make_chunk_inputs(w, random_state=True), TOL_F32, chunk=chunk)


def test_simt_bf16_varlen():
    w = Workload("s", B=1, T=0, H=2, d_k=64, d_v=96, dtype=torch.bfloat16, seed=6)
    check(make_chunk_inputs(w, lengths=[33, 0, 90, 1], random_state=True), TOL_BF16, chunk=32)


def test_simt_chunk_size_independence():
    w = Workload("s", B=1, T=150, H=2, d_k=64, d_v=64, dtype=torch.float32, seed=8)
    inp = make_chunk_inputs(w, random_state=True)
    outs = [gpu_chunk(inp, chunk=c) for c in (16, 32, 64)]
    for o, fs in outs[1:]:
        assert rel_l2(np64(o), np64(outs[0][0])) < 1e-5
        assert rel_l2(np64(fs), np64(outs[0][1])) < 1e-5


# ---------------------------------------------------------------- segmented state scan
def _segments(inp):
    import gated_delta_rule_112_b200 as gdn
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return gdn.lib().gdn_chunk_fwd_scan_segments(inp["B"], inp["T"], inp["H"], 128, 128, 0, 64,
                                                 gdn.BF16, sms)


def test_tc_segmented_scan_one_head_ragged_tail():
    inp = make_chunk_inputs(SMALL, B=1, H=1, T=64 * 40 + 37, random_state=True)
    assert _segments(inp) > 1
    check(inp, TOL_BF16)


def test_tc_segmented_scan_batch_heads_slow_decay():
    inp = make_chunk_inputs(SMALL, B=2, H=2, T=64 * 47, random_state=True, gate_mu=-4.0)
    assert _segments(inp) > 1
    check(inp, TOL_BF16)


def test_tc_segmented_scan_without_final_state_or_initial_state():
    import gated_delta_rule_112_b200 as gdn
    inp = make_chunk_inputs(SMALL, B=1, H=2, T=64 * 33)
    assert _segments(inp) > 1
    d = to_dev(inp)
    o, fs = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, None,
                          output_final_state=False)
    torch.cuda.synchronize()
    assert fs is None
    ro, _ = oracle_chunk(inp)
    assert_close("o", np64(o), ro, TOL_BF16)


# ---------------------------------------------------------------- the workloads
def test_workload_tiny_fp32():
    check(make_chunk_inputs("tiny_fp32"), TOL_F32)


def test_workload_b4h16t4096():
    check(make_chunk_inputs("b4h16t4096"), TOL_BF16)


def test_workload_long64k():
    """B=1 H=16 T=65536 (random S_0, slow decay), every head against the oracle."""
    check(make_chunk_inputs("long64k"), TOL_BF16)


def test_workload_beta_up_to_two():
    """b4h16t4096 with beta in (0, 2) (I - beta k k^T has a negative eigenvalue
    for beta > 1), every head against the oracle."""
    inp = make_chunk_inputs("b4h16t4096_beta2")
    assert float(inp["beta"].max()) > 1.9
    check(inp, TOL_BF16)


def test_workload_varlen64():
    """64 packed sequences (38,268 tokens), H=32, every head against the oracle."""
    check(make_chunk_inputs("varlen64"), TOL_BF16)

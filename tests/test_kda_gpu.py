"""GPU parity of the channel-wise-gate (KDA) entry points -- gdn_kda_chunk_fwd
and gdn_kda_decode_step -- against the fp64 oracle on the same seeded inputs,
through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_112_b200.inputs import Workload, make_chunk_inputs, make_decode_inputs
from tests.parity import TOL_BF16, TOL_F32, assert_close, np64, rel_l2, to_dev

pytestmark = pytest.mark.gpu

SMALL = Workload("kda_small", B=1, T=64, H=1, d_k=128, d_v=128, seed=21, gate="channel",
                 dtype=torch.float32)


def oracle_kda(inp, heads=None):
    sl = slice(None) if heads is None else heads
    s0, cu = inp["initial_state"], inp["cu_seqlens"]
    return oracle.kda_chunk_fwd(np64(inp["q"][:, :, sl]), np64(inp["k"][:, :, sl]),
                                np64(inp["v"][:, :, sl]), np64(inp["g"][:, :, sl]),
                                np64(inp["beta"][:, :, sl]),
                                None if s0 is None else np64(s0[:, sl]),
                                None if cu is None else cu.numpy())


def gpu_kda(inp, chunk=None):
    import gated_delta_rule_112_b200 as gdn
    d = to_dev(inp)
    o, fs = gdn.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"],
                              d["cu_seqlens"], chunk=chunk or inp["chunk"])
    torch.cuda.synchronize()
    return o, fs


def check(inp, tol, chunk=None, heads=None):
    o, fs = gpu_kda(inp, chunk)
    ro, rfs = oracle_kda(inp, heads)
    if heads is not None:
        o, fs = o[:, :, heads], fs[:, heads]
    assert_close("o", np64(o), ro, tol)
    assert_close("final_state", np64(fs), rfs, tol)
    return o, fs


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 63, 65, 200])
def test_kda_fp32_ragged_lengths_and_chunks(chunk, T):
    check(make_chunk_inputs(SMALL, T=T, H=2, random_state=True), TOL_F32, chunk=chunk)


@pytest.mark.parametrize("dk,dv", [(64, 48), (128, 32), (96, 128)])
def test_kda_fp32_head_sizes(dk, dv):
    w = Workload("kda_sizes", B=2, T=150, H=2, d_k=dk, d_v=dv, seed=22, gate="channel",
                 dtype=torch.float32, random_state=True)
    check(make_chunk_inputs(w), TOL_F32, chunk=32)


def test_kda_bf16_varlen_odd_lengths_with_states():
    inp = make_chunk_inputs(SMALL, H=2, lengths=[70, 1, 130, 64, 5], random_state=True,
                            dtype=torch.bfloat16)
    check(inp, TOL_BF16)


# ---------------------------------------------------------------- tensor-core path
KDA_TC = Workload("kda_tc", B=1, T=64, H=1, d_k=128, d_v=128, seed=24, gate="channel")


def test_kda_tc_path_is_selected():
    import gated_delta_rule_112_b200 as gdn
    assert gdn.chunk_path(128, 128, 64, torch.bfloat16) == gdn.PATH_TCGEN05
    tc = gdn.lib().gdn_kda_chunk_fwd_workspace_size(1, 64, 1, 128, 128, 0, 64, gdn.BF16)
    simt = gdn.lib().gdn_kda_chunk_fwd_workspace_size(1, 64, 1, 128, 128, 0, 64, gdn.F32)
    assert tc > simt          # the tensor-core layout holds the per-chunk operand tiles
    # The tensor-core kernels run the chunk on bf16 operand tiles, so the state
    # carries their rounding; the fp32 CUDA-core kernel agrees with the fp64
    # oracle to about 1e-6. Both stay within the bf16 tolerance.
    inp = make_chunk_inputs(KDA_TC, T=200, H=2, random_state=True)
    _, fs = gpu_kda(inp)
    _, rfs = oracle_kda(inp)
    assert 2e-5 < rel_l2(np64(fs), rfs) < TOL_BF16


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_kda_tc_ragged_lengths(T):
    check(make_chunk_inputs(KDA_TC, T=T, H=2, random_state=True), TOL_BF16)


def test_kda_tc_batch_heads_with_initial_state():
    check(make_chunk_inputs(KDA_TC, B=3, H=3, T=257, random_state=True), TOL_BF16)


def test_kda_tc_strong_decay():
    # log alpha ~ -softplus(N(3, 1)) per token and channel: within a chunk the
    # decay reaches exp(-200); the block-scaled factors stay within fp32.
    check(make_chunk_inputs(KDA_TC, B=2, H=2, T=192, random_state=True, gate_mu=3.0), TOL_BF16)


def test_kda_tc_segmented_scan():
    import gated_delta_rule_112_b200 as gdn
    inp = make_chunk_inputs(KDA_TC, B=1, H=1, T=64 * 40 + 37, random_state=True)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert gdn.lib().gdn_chunk_fwd_scan_segments(1, inp["T"], 1, 128, 128, 0, 64, gdn.BF16,
                                                 sms) > 1
    check(inp, TOL_BF16)


def test_kda_tc_equal_channels_match_the_scalar_gate():
    import gated_delta_rule_112_b200 as gdn
    inp = make_chunk_inputs(KDA_TC, B=2, H=2, T=160, random_state=True)
    gs = inp["g"][..., 0].contiguous()
    inp["g"] = gs[..., None].expand(-1, -1, -1, 128).contiguous()
    o1, f1 = gpu_kda(inp)
    d = to_dev(inp)
    o2, f2 = gdn.chunk_fwd(d["q"], d["k"], d["v"], gs.cuda(), d["beta"], d["initial_state"])
    torch.cuda.synchronize()
    # both on bf16 tensor-core tiles, with different roundings of the decays
    assert rel_l2(np64(o1), np64(o2)) < TOL_BF16
    assert rel_l2(np64(f1), np64(f2)) < TOL_BF16


def test_kda_empty_sequences_keep_their_state():
    inp = make_chunk_inputs(SMALL, H=2, lengths=[0, 40, 0, 3], random_state=True)
    o, fs = check(inp, TOL_F32)
    s0 = inp["initial_state"]
    np.testing.assert_array_equal(np64(fs[0]), np64(s0[0]))
    np.testing.assert_array_equal(np64(fs[2]), np64(s0[2]))


def test_kda_zero_tokens():
    inp = make_chunk_inputs(SMALL, B=2, H=2, T=0, random_state=True)
    o, fs = gpu_kda(inp)
    assert o.shape == (2, 0, 2, 128)
    np.testing.assert_array_equal(np64(fs), np64(inp["initial_state"]))


def test_kda_strong_decay_stays_finite_and_exact():
    # log alpha = -softplus(N(3, 1)) ~ -3 per token and channel: within a chunk
    # of 64 the cumulative decay reaches exp(-200); every factor the kernel
    # forms is exp of a difference over tokens in between, so nothing overflows.
    inp = make_chunk_inputs(SMALL, B=2, H=2, T=192, random_state=True, gate_mu=3.0)
    check(inp, TOL_F32)


def test_kda_equal_channels_matches_scalar_gate_path():
    import gated_delta_rule_112_b200 as gdn
    inp = make_chunk_inputs(SMALL, B=2, H=2, T=160, random_state=True)
    gs = inp["g"][..., 0].contiguous()
    inp["g"] = gs[..., None].expand(-1, -1, -1, 128).contiguous()
    o1, f1 = gpu_kda(inp)
    d = to_dev(inp)
    o2, f2 = gdn.chunk_fwd(d["q"], d["k"], d["v"], gs.cuda(), d["beta"], d["initial_state"],
                           chunk=64, force_simt=True)
    assert rel_l2(np64(o1), np64(o2)) < 1e-6
    assert rel_l2(np64(f1), np64(f2)) < 1e-6


def test_workload_kda_b4h16t4096():
    """The kda_b4h16t4096 workload (B=4, T=4096, H=16, d=128, bf16) at full size
    in one call, as the benchmark runs it; every head against the oracle."""
    inp = make_chunk_inputs("kda_b4h16t4096")
    o, fs = gpu_kda(inp)
    ro, rfs = oracle_kda(inp)
    assert_close("o", np64(o), ro, TOL_BF16)
    assert_close("final_state", np64(fs), rfs, TOL_BF16)


# ---------------------------------------------------------------- decode
def run_steps(d, steps):
    import gated_delta_rule_112_b200 as gdn
    st = d["state"].cuda()
    outs = []
    for t in range(steps):
        o = gdn.kda_decode_step(d["q"][t].cuda(), d["k"][t].cuda(), d["v"][t].cuda(),
                                d["g"][t].cuda(), d["beta"][t].cuda(), st)
        outs.append(o.float().cpu())
    torch.cuda.synchronize()
    return outs, st.cpu()


def oracle_steps(d, steps, units=None):
    st = np64(d["state"])
    if units is not None:
        st = st[units[0], units[1]][:, None]
    outs = []
    for t in range(steps):
        q, k, v, g, b = (np64(d[key][t]) for key in ("q", "k", "v", "g", "beta"))
        if units is not None:
            q, k, v, g, b = (x[units[0], units[1]][:, None] for x in (q, k, v, g, b))
        o, st = oracle.kda_decode_step(q, k, v, g, b, st)
        outs.append(o)
    return outs, st


@pytest.mark.parametrize("dtype,dk,dv,tol", [(torch.bfloat16, 128, 128, TOL_BF16),
                                             (torch.float32, 128, 128, TOL_F32),
                                             (torch.float32, 64, 32, TOL_F32)])
def test_kda_decode_small_chained(dtype, dk, dv, tol):
    w = Workload("t", B=5, T=1, H=3, d_k=dk, d_v=dv, dtype=dtype, random_state=True, seed=23,
                 steps=4, gate="channel")
    d = make_decode_inputs(w)
    got, st = run_steps(d, 4)
    ref, rst = oracle_steps(d, 4)
    for t in range(4):
        assert_close(f"o step {t}", got[t].numpy(), ref[t], tol)
    assert_close("state", st.numpy(), rst, tol)


def test_workload_kda_decode_full_size():
    """kda_decode (N=256, H=32, 64 steps): every state and output against the oracle."""
    d = make_decode_inputs("kda_decode")
    steps = d["steps"]
    got, st = run_steps(d, steps)
    ref, rst = oracle_steps(d, steps)
    assert_close("o all 64 steps", np.stack([g.numpy() for g in got]), np.stack(ref), TOL_BF16)
    assert_close("state after 64 steps", st.numpy(), rst, TOL_BF16)


def test_kda_rejects_scalar_shaped_gate():
    import gated_delta_rule_112_b200 as gdn
    inp = make_chunk_inputs(SMALL, T=64)
    d = to_dev(inp)
    with pytest.raises(ValueError):
        gdn.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"][..., 0].contiguous(), d["beta"])

"""GPU parity of gdn_chunk_bwd (the gradients of the forward pass) against the
fp64 oracle ``oracle.chunk_bwd`` on the same seeded inputs, through the C ABI.

Two paths. The token-level backward (gdn_chunk_bwd_exact, and gdn_chunk_bwd
for fp32 inputs or other head sizes) computes in fp32 from the given inputs
(bf16 inputs are upcast exactly, as the oracle sees them); a CPU emulation of
its arithmetic in fp32 stays within 3e-7 of the fp64 gradients, so the fp32
tolerance applies to both input types. The chunkwise tensor-core backward
(gdn_chunk_bwd for bf16 with d_k = d_v = 128) multiplies bf16 operands with
fp32 accumulation, as the forward's tensor-core path does, and is held to the
bf16 tolerance."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_112_b200.inputs import Workload, make_chunk_inputs
from tests.parity import TOL_BF16, TOL_F32, assert_close, np64, oracle_chunk, to_dev

pytestmark = pytest.mark.gpu

SMALL = Workload("bwd_small", B=2, T=64, H=2, d_k=128, d_v=128, seed=31, dtype=torch.float32)
KEYS = ("dq", "dk", "dv", "dg", "dbeta", "d_initial_state")


def upstream(inp, seed=0, with_dsN=True):
    gen = torch.Generator("cpu").manual_seed(seed)
    B, T, H, dv = inp["B"], inp["T"], inp["H"], inp["d_v"]
    d_o = torch.randn(B, T, H, dv, generator=gen).to(inp["dtype"])
    N = inp["num_seqs"]
    dsN = 0.1 * torch.randn(N, H, inp["d_k"], dv, generator=gen) if with_dsN else None
    return d_o, dsN


def check(inp, d_o, dsN, tol=TOL_F32, heads=None, exact=False):
    import gated_delta_rule_112_b200 as gdn
    d = to_dev(inp)
    got = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d_o.cuda(),
                        d["initial_state"], d["cu_seqlens"],
                        None if dsN is None else dsN.cuda(), exact=exact)
    torch.cuda.synchronize()
    assert gdn.get_status() == gdn.OK
    sl = slice(None) if heads is None else heads
    s0, cu = inp["initial_state"], inp["cu_seqlens"]
    ref = oracle.chunk_bwd(np64(inp["q"][:, :, sl]), np64(inp["k"][:, :, sl]),
                           np64(inp["v"][:, :, sl]), np64(inp["g"][:, :, sl]),
                           np64(inp["beta"][:, :, sl]), np64(d_o[:, :, sl]),
                           None if s0 is None else np64(s0[:, sl]),
                           None if cu is None else cu.numpy(),
                           None if dsN is None else np64(dsN[:, sl]))
    for key in KEYS:
        g = got[key]
        g = g[:, sl] if key == "d_initial_state" else g[:, :, sl]
        assert_close(key, np64(g), ref[key], tol)
    return got


@pytest.mark.parametrize("T", [1, 7, 130])
@pytest.mark.parametrize("with_state", [False, True])
def test_bwd_fp32_lengths(T, with_state):
    inp = make_chunk_inputs(SMALL, T=T, random_state=with_state)
    d_o, dsN = upstream(inp, seed=T, with_dsN=with_state)
    check(inp, d_o, dsN)


@pytest.mark.parametrize("dk,dv", [(64, 32), (96, 128), (128, 64), (128, 96), (64, 80)])
def test_bwd_fp32_head_sizes(dk, dv):
    w = Workload("bwd_sizes", B=2, T=90, H=2, d_k=dk, d_v=dv, seed=32, dtype=torch.float32,
                 random_state=True)
    inp = make_chunk_inputs(w)
    d_o, dsN = upstream(inp, seed=1)
    check(inp, d_o, dsN)


def test_bwd_bf16_varlen_with_empty_sequences():
    inp = make_chunk_inputs(SMALL, lengths=[50, 0, 131, 1], random_state=True,
                            dtype=torch.bfloat16)
    d_o, dsN = upstream(inp, seed=2)
    got = check(inp, d_o, dsN, exact=True)
    # an empty sequence passes the final-state gradient straight through
    np.testing.assert_array_equal(np64(got["d_initial_state"][1]), np64(dsN[1]))


def test_bwd_zero_tokens():
    import gated_delta_rule_112_b200 as gdn
    inp = make_chunk_inputs(SMALL, T=0, random_state=True)
    d_o, dsN = upstream(inp, seed=3)
    d = to_dev(inp)
    got = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d_o.cuda(),
                        d["initial_state"], None, dsN.cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(np64(got["d_initial_state"]), np64(dsN))


def test_bwd_bad_cu_seqlens_reported():
    import gated_delta_rule_112_b200 as gdn
    inp = make_chunk_inputs(SMALL, lengths=[5, 5, 5], random_state=True)
    d_o, dsN = upstream(inp, seed=4)
    d = to_dev(inp)
    bad = torch.tensor([0, 9, 4, 15], dtype=torch.int32, device="cuda")   # decreasing
    ws = torch.empty(gdn.bwd_workspace_size(1, 15, 2, 128, 128, 3, torch.float32),
                     dtype=torch.uint8, device="cuda")
    gdn.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d_o.cuda(), d["initial_state"],
                  bad, dsN.cuda(), workspace=ws)
    assert gdn.get_status(ws) == gdn.ERR_INVALID_ARG
    assert gdn.get_status(ws) == gdn.OK          # the word is cleared


def test_bwd_exact_full_size_workload_sampled_heads():
    """The b4h16t4096 workload (bf16, B=4, T=4096, H=16, d=128) in one call of
    the token-level path; the oracle differentiates two heads of every sequence."""
    inp = make_chunk_inputs("b4h16t4096")
    d_o, dsN = upstream(inp, seed=5)
    check(inp, d_o, dsN, heads=[2, 9], exact=True)


# ---------------------------------------------------- chunkwise tensor-core path
TC = Workload("bwd_tc", B=2, T=64, H=2, d_k=128, d_v=128, seed=33)


def test_bwd_tc_path_is_the_default_for_bf16_d128():
    import gated_delta_rule_112_b200 as gdn
    tc = gdn.bwd_workspace_size(4, 4096, 16, 128, 128)
    exact = gdn.bwd_workspace_size(4, 4096, 16, 128, 128, exact=True)
    assert tc < exact / 30           # O(T/64 d^2) against O(T d^2)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
@pytest.mark.parametrize("with_state", [False, True])
def test_bwd_tc_lengths(T, with_state):
    inp = make_chunk_inputs(TC, T=T, random_state=with_state)
    d_o, dsN = upstream(inp, seed=40 + T, with_dsN=with_state)
    check(inp, d_o, dsN, tol=TOL_BF16)


def test_bwd_tc_batch_heads():
    inp = make_chunk_inputs(TC, B=3, H=5, T=257, random_state=True)
    d_o, dsN = upstream(inp, seed=41)
    check(inp, d_o, dsN, tol=TOL_BF16)


def test_bwd_tc_varlen_with_empty_sequences():
    inp = make_chunk_inputs(TC, H=2, lengths=[50, 0, 131, 1, 64], random_state=True)
    d_o, dsN = upstream(inp, seed=42)
    got = check(inp, d_o, dsN, tol=TOL_BF16)
    np.testing.assert_array_equal(np64(got["d_initial_state"][1]), np64(dsN[1]))


def test_bwd_tc_strong_decay_and_large_beta():
    """gamma underflows inside a chunk (g ~ -softplus(N(3, 1))) and beta in
    (0, 2): the recomputed decays and the division-free dbeta stay finite."""
    w = Workload("bwd_tc_hard", B=2, T=64, H=2, d_k=128, d_v=128, seed=34, beta_scale=2.0)
    inp = make_chunk_inputs(w, T=192, random_state=True, gate_mu=3.0)
    d_o, dsN = upstream(inp, seed=43)
    check(inp, d_o, dsN, tol=TOL_BF16)


def test_bwd_tc_zero_beta_rows():
    """beta = 0 on some tokens: A and U lose those rows, T diag(beta) those
    columns; dbeta there is still the residual product, with no division."""
    inp = make_chunk_inputs(TC, T=130, random_state=True)
    inp["beta"][:, ::3] = 0.0
    d_o, dsN = upstream(inp, seed=44)
    check(inp, d_o, dsN, tol=TOL_BF16)


def test_bwd_tc_zero_tokens():
    import gated_delta_rule_112_b200 as gdn
    inp = make_chunk_inputs(TC, T=0, random_state=True)
    d_o, dsN = upstream(inp, seed=45)
    d = to_dev(inp)
    got = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d_o.cuda(),
                        d["initial_state"], None, dsN.cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(np64(got["d_initial_state"]), np64(dsN))


def test_workload_bwd_b4h16t4096():
    """The full b4h16t4096 step on the tensor-core path, every head and every
    gradient against the oracle."""
    inp = make_chunk_inputs("b4h16t4096")
    d_o, dsN = upstream(inp, seed=5)
    check(inp, d_o, dsN, tol=TOL_BF16)


def check_saved(inp, d_o, dsN):
    """A training step through chunk_fwd_save and chunk_bwd_saved: the forward
    outputs and all six gradients against the oracle, the gradients also
    against the replaying chunk_bwd (the saved intermediates and chunk states
    are the ones the replay recomputes), and a second backward from the same
    saved workspace unchanged."""
    import gated_delta_rule_112_b200 as gdn
    d = to_dev(inp)
    fwd = (d["q"], d["k"], d["v"], d["g"], d["beta"])
    dsn = None if dsN is None else dsN.cuda()
    o, fs, saved = gdn.chunk_fwd_save(*fwd, d["initial_state"], d["cu_seqlens"])
    torch.cuda.synchronize()
    assert gdn.get_status() == gdn.OK
    ref_o, ref_s = oracle_chunk(inp)
    assert_close("o", np64(o), ref_o, TOL_BF16)
    assert_close("final_state", np64(fs), ref_s, TOL_BF16)
    got = gdn.chunk_bwd_saved(*fwd, d_o.cuda(), saved, d["initial_state"], d["cu_seqlens"], dsn)
    again = gdn.chunk_bwd_saved(*fwd, d_o.cuda(), saved, d["initial_state"], d["cu_seqlens"],
                                dsn)
    replay = gdn.chunk_bwd(*fwd, d_o.cuda(), d["initial_state"], d["cu_seqlens"], dsn)
    torch.cuda.synchronize()
    assert gdn.get_status() == gdn.OK
    s0, cu = inp["initial_state"], inp["cu_seqlens"]
    ref = oracle.chunk_bwd(np64(inp["q"]), np64(inp["k"]), np64(inp["v"]), np64(inp["g"]),
                           np64(inp["beta"]), np64(d_o), None if s0 is None else np64(s0),
                           None if cu is None else cu.numpy(),
                           None if dsN is None else np64(dsN))
    for key in KEYS:
        assert_close(key, np64(got[key]), ref[key], TOL_BF16)
        if key in ("dg", "dbeta"):
            # summed from per-warp partials by shared-memory atomics: equal
            # across calls to rounding, not bit for bit
            assert_close(key + " (repeat)", np64(again[key]), np64(got[key]), 1e-6)
        else:
            assert torch.equal(got[key], again[key]), key
        # the same kernels on the same intermediates as the replay
        assert_close(key + " (saved vs replay)", np64(got[key]), np64(replay[key]), 1e-5)
    return got


def test_bwd_saved_batch_heads():
    inp = make_chunk_inputs(TC, B=3, H=5, T=257, random_state=True)
    d_o, dsN = upstream(inp, seed=46)
    check_saved(inp, d_o, dsN)


def test_bwd_saved_varlen_with_empty_sequences():
    inp = make_chunk_inputs(TC, H=2, lengths=[50, 0, 131, 1, 64], random_state=True)
    d_o, dsN = upstream(inp, seed=47)
    got = check_saved(inp, d_o, dsN)
    np.testing.assert_array_equal(np64(got["d_initial_state"][1]), np64(dsN[1]))


def test_bwd_saved_zero_tokens():
    import gated_delta_rule_112_b200 as gdn
    inp = make_chunk_inputs(TC, T=0, random_state=True)
    d_o, dsN = upstream(inp, seed=48)
    d = to_dev(inp)
    fwd = (d["q"], d["k"], d["v"], d["g"], d["beta"])
    o, fs, saved = gdn.chunk_fwd_save(*fwd, d["initial_state"])
    got = gdn.chunk_bwd_saved(*fwd, d_o.cuda(), saved, d["initial_state"], None, dsN.cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(np64(fs), np64(inp["initial_state"]))
    np.testing.assert_array_equal(np64(got["d_initial_state"]), np64(dsN))


def test_bwd_saved_rejects_other_paths():
    import gated_delta_rule_112_b200 as gdn
    inp = make_chunk_inputs(SMALL, T=64)          # fp32: the token-level backward's domain
    d = to_dev(inp)
    with pytest.raises(gdn.GdnError):
        gdn.chunk_fwd_save(d["q"], d["k"], d["v"], d["g"], d["beta"])

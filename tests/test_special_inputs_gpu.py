"""Tensor-core path on the inputs whose answers the recurrence fixes in closed
form (the special cases the pages' formula reduces to), compared with those
closed forms and with the fp64 oracle, through the C ABI.

The recurrence (phantomic12 "gated-deltanet" page, mechanism paragraph; dmarx
anthology LIT-137, "Standing in the anthology"):
S_t = S_{t-1} alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t.
  * beta = 0: pure decay, S_t = exp(Gamma_t) S_0, o_t = exp(Gamma_t) S_0 q_t
  * g = 0 (alpha = 1): the ungated delta rule
  * |k_t| = 1, beta_t = 1: the write overwrites the value bound to k_t, so
    S_t k_t = v_t for any alpha and any earlier state; with q_t = k_t every
    output equals its own value, o_t = v_t
  * strong decay (log alpha ~ -softplus(N(3, 1)), about -3 per token): the
    within-chunk decay factors underflow fp32 inside one 64-token chunk
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_112_b200.inputs import Workload, make_chunk_inputs
from tests.parity import TOL_BF16, assert_close, gpu_chunk, np64, oracle_chunk

pytestmark = pytest.mark.gpu

BASE = Workload("special", B=2, T=300, H=3, d_k=128, d_v=128, seed=41, random_state=True)


def _check_oracle(inp, o, fs):
    ro, rfs = oracle_chunk(inp)
    assert_close("o vs oracle", np64(o), ro, TOL_BF16)
    assert_close("final_state vs oracle", np64(fs), rfs, TOL_BF16)


def test_tc_beta_zero_is_pure_decay():
    inp = make_chunk_inputs(BASE)
    inp["beta"] = torch.zeros_like(inp["beta"])
    o, fs = gpu_chunk(inp)
    # closed form, in the stored orientation state[n][h][j][i] = S_ij
    s0 = np64(inp["initial_state"])                  # [N,H,dk,dv]
    G = np.cumsum(np64(inp["g"]), axis=1)            # Gamma_t, [B,T,H]
    q = np64(inp["q"])
    ref_o = np.exp(G)[..., None] * np.einsum("bhji,bthj->bthi", s0, q)
    ref_s = np.exp(G[:, -1])[:, :, None, None] * s0
    assert_close("o vs closed form", np64(o), ref_o, TOL_BF16)
    assert_close("final_state vs closed form", np64(fs), ref_s, TOL_BF16)
    _check_oracle(inp, o, fs)


def test_tc_gate_zero_is_ungated_delta_rule():
    inp = make_chunk_inputs(BASE)
    inp["g"] = torch.zeros_like(inp["g"])
    o, fs = gpu_chunk(inp)
    _check_oracle(inp, o, fs)


def _unit_keys(shape, gen):
    """Keys of exactly unit norm in bf16: four entries of +-1/2 at distinct
    random positions (0.5 and its square are exact in every format)."""
    *lead, d = shape
    n = int(np.prod(lead))
    k = torch.zeros(n, d)
    pos = torch.argsort(torch.rand(n, d, generator=gen), dim=1)[:, :4]
    sign = torch.where(torch.rand(n, 4, generator=gen) < 0.5, -0.5, 0.5)
    k.scatter_(1, pos, sign)
    return k.reshape(shape)


def test_tc_unit_keys_beta_one_overwrite():
    inp = make_chunk_inputs(BASE)
    gen = torch.Generator("cpu").manual_seed(42)
    k = _unit_keys(tuple(inp["k"].shape), gen).to(torch.bfloat16)
    assert torch.all(k.float().pow(2).sum(-1) == 1.0)
    inp["k"] = k.contiguous()
    inp["q"] = k.clone().contiguous()                  # read back the key just written
    inp["beta"] = torch.ones_like(inp["beta"])
    o, fs = gpu_chunk(inp)
    v = np64(inp["v"])
    # o_t = S_t k_t = v_t for every token
    assert_close("o vs v (overwrite)", np64(o), v, TOL_BF16)
    # S_T k_T = v_T on the final state
    sk = np.einsum("bhji,bhj->bhi", np64(fs), np64(inp["k"][:, -1]))
    assert_close("S_T k_T vs v_T", sk, v[:, -1], TOL_BF16)
    _check_oracle(inp, o, fs)


def test_tc_strong_decay_underflows_inside_a_chunk():
    inp = make_chunk_inputs(BASE, gate_mu=3.0)
    # the decay over some 64-token chunk is below the smallest fp32 value
    g = inp["g"].double()
    per_chunk = g[:, :256].reshape(g.shape[0], 4, 64, g.shape[2]).sum(2)
    assert float(per_chunk.max()) < -104.0
    o, fs = gpu_chunk(inp)
    _check_oracle(inp, o, fs)

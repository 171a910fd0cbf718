"""Pins for the channel-wise-gate oracle (the Kimi Delta Attention variant of
the recurrence: one decay per d_k channel), each against something other than
that oracle.

The pages name the variant only as replacing the scalar decay with a
channel-wise one (dmarx anthology LIT-137, "Standing in the anthology";
SOTA-135, "Sequence"). The reading: diag(alpha_t) stands where the scalar
alpha_t stood, S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
The tests check that oracle against a hand-worked exact example, the scalar
gate it must reduce to (pinned on its own), closed forms for pure decay and
for an overwriting unit key, and an independent chunkwise formulation with
the decay inside the dot products. A decay on the wrong axis, a residual read
from the undecayed state, the decay applied after the write or a dropped gate
fails at least one of them (tests/test_oracle_mutations.py plants each).
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle.chunked import kda_chunk_fwd_dense

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def make(seed, B=1, T=7, H=2, dk=5, dv=3, s0=True, mu=-1.0, sigma=1.0):
    r = np.random.default_rng(seed)
    q = unit(r.standard_normal((B, T, H, dk)))
    k = unit(r.standard_normal((B, T, H, dk)))
    v = r.standard_normal((B, T, H, dv))
    g = -np.log1p(np.exp(sigma * r.standard_normal((B, T, H, dk)) + mu))
    beta = r.uniform(0.05, 1.0, (B, T, H))
    S0 = 0.3 * r.standard_normal((B, H, dk, dv)) if s0 else None
    return q, k, v, g, beta, S0


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def _golden():
    fx = json.load(open(os.path.join(GOLDEN, "kda_hand_t2_dk2_dv3.json")))
    k = np.array(fx["k"], float)[None, :, None, :]
    q = np.array(fx["q"], float)[None, :, None, :]
    v = np.array(fx["v"], float)[None, :, None, :]
    g = np.log(np.array(fx["alpha"], float))[None, :, None, :]
    beta = np.array(fx["beta"], float)[None, :, None]
    s0 = np.array(fx["initial_state"], float)[None, None]
    return fx, q, k, v, g, beta, s0


def test_kda_hand_worked_two_tokens():
    fx, q, k, v, g, beta, s0 = _golden()
    o, fs = oracle.kda_chunk_fwd(q, k, v, g, beta, s0)
    np.testing.assert_allclose(o[0, :, 0], np.array(fx["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(fs[0, 0], np.array(fx["final_state"]), rtol=0, atol=1e-14)
    o2, fs2 = kda_chunk_fwd_dense(q, k, v, g, beta, s0, chunk=2)
    np.testing.assert_allclose(o2[0, :, 0], np.array(fx["o"]), atol=1e-14)
    np.testing.assert_allclose(fs2[0, 0], np.array(fx["final_state"]), atol=1e-14)


def test_kda_decode_step_matches_hand_worked_first_token():
    fx, q, k, v, g, beta, s0 = _golden()
    o, st = oracle.kda_decode_step(q[0, :1], k[0, :1], v[0, :1], g[0, :1], beta[0, :1],
                                   s0[:, :1])
    np.testing.assert_allclose(o[0, 0], np.array(fx["o"][0]), rtol=0, atol=1e-14)
    # after token 1 of the derivation: S_1 = [[7/8,3/8],[-1/8,3/8],[21/16,17/16]]
    s1 = np.array([[7 / 8, 3 / 8], [-1 / 8, 3 / 8], [21 / 16, 17 / 16]])
    np.testing.assert_allclose(st[0, 0], s1.T, rtol=0, atol=1e-14)


def test_kda_equal_channels_is_scalar_gate():
    q, k, v, g, beta, S0 = make(1, T=23, dk=6, dv=4)
    gs = g[..., 0]
    o1, f1 = oracle.chunk_fwd(q, k, v, gs, beta, S0)
    o2, f2 = oracle.kda_chunk_fwd(q, k, v, np.repeat(gs[..., None], 6, axis=-1), beta, S0)
    assert rel(o2, o1) < 1e-13 and rel(f2, f1) < 1e-13


def test_kda_beta_zero_is_channel_decay():
    # beta = 0: S_t = S_0 diag(prod alpha), o_t = S_0 diag(exp(Gamma_t)) q_t; the
    # decay scales the state's d_k axis (memory rows j of state[j][i]).
    q, k, v, g, beta, S0 = make(2, T=9, dk=4, dv=3)
    beta[:] = 0.0
    o, fs = oracle.kda_chunk_fwd(q, k, v, g, beta, S0)
    Gam = np.cumsum(g[0], axis=0)                         # [T, H, dk]
    for h in range(2):
        want_fs = S0[0, h] * np.exp(Gam[-1, h])[:, None]
        np.testing.assert_allclose(fs[0, h], want_fs, rtol=1e-13, atol=1e-15)
        for t in range(9):
            want_o = S0[0, h].T @ (np.exp(Gam[t, h]) * q[0, t, h])
            np.testing.assert_allclose(o[0, t, h], want_o, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("m", [0, 3])
def test_kda_unit_key_beta_one_overwrites(m):
    # one token, k = e_m, beta = 1: column m of S_1 is v exactly, every other
    # column j is alpha_j times its old value (the decay acts before the write).
    q, k, v, g, beta, S0 = make(3, T=1, H=1, dk=5, dv=4)
    k[:] = 0.0
    k[0, 0, 0, m] = 1.0
    beta[:] = 1.0
    o, fs = oracle.kda_chunk_fwd(q, k, v, g, beta, S0)
    alpha = np.exp(g[0, 0, 0])
    want = S0[0, 0] * alpha[:, None]
    want[m] = v[0, 0, 0]
    np.testing.assert_allclose(fs[0, 0], want, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(o[0, 0, 0], want.T @ q[0, 0, 0], rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("chunk", [1, 4, 16])
@pytest.mark.parametrize("T", [1, 7, 21])
def test_kda_dense_chunked_matches_token_loop(chunk, T):
    q, k, v, g, beta, S0 = make(4 + T, T=T, dk=6, dv=5, mu=0.5, sigma=2.0)
    o1, f1 = oracle.kda_chunk_fwd(q, k, v, g, beta, S0)
    o2, f2 = kda_chunk_fwd_dense(q, k, v, g, beta, S0, chunk=chunk)
    assert rel(o2, o1) < 1e-11 and rel(f2, f1) < 1e-11


def test_kda_varlen_equals_separate_sequences():
    lens = [5, 0, 12, 3]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k, v, g, beta, _ = make(5, T=int(cu[-1]), dk=4, dv=3)
    S0 = 0.3 * np.random.default_rng(6).standard_normal((len(lens), 2, 4, 3))
    o, fs = oracle.kda_chunk_fwd(q, k, v, g, beta, S0, cu_seqlens=cu)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        on, fn = oracle.kda_chunk_fwd(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b],
                                      beta[:, a:b], S0[n:n + 1])
        np.testing.assert_allclose(o[:, a:b], on, rtol=0, atol=1e-14)
        np.testing.assert_allclose(fs[n], fn[0], rtol=0, atol=1e-14)


def test_kda_rejects_scalar_shaped_gate():
    q, k, v, g, beta, S0 = make(7)
    with pytest.raises(ValueError):
        oracle.kda_chunk_fwd(q, k, v, g[..., 0], beta, S0)


def test_kda_linear_in_values_and_state():
    # S_t and o_t are jointly linear in (V, S_0) for fixed keys, queries and gates
    q, k, v, g, beta, S0 = make(8, T=15, dk=4, dv=3)
    o1, f1 = oracle.kda_chunk_fwd(q, k, v, g, beta, S0)
    o2, f2 = oracle.kda_chunk_fwd(q, k, -2.5 * v, g, beta, -2.5 * S0)
    np.testing.assert_allclose(o2, -2.5 * o1, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(f2, -2.5 * f1, rtol=1e-13, atol=1e-14)


def test_kda_cycling_unit_keys_closed_form():
    # k_t = e_{t mod d_k}, beta = 1: each token first decays every column of S by
    # its own channel's alpha, then overwrites column t mod d_k with v_t. So
    # column m of S_T is v_tau times the decays of channel m after tau (tau = the
    # last token that wrote it), or S_0's column times all its decays.
    dk, dv, T = 4, 3, 10
    q, k, v, g, beta, S0 = make(9, T=T, H=1, dk=dk, dv=dv)
    k[:] = 0.0
    for t in range(T):
        k[0, t, 0, t % dk] = 1.0
    beta[:] = 1.0
    _, fs = oracle.kda_chunk_fwd(q, k, v, g, beta, S0)
    alpha = np.exp(g[0, :, 0])                   # [T, dk]
    want = np.zeros((dk, dv))                    # S^T storage: row m = column m of S
    for m in range(dk):
        writers = [t for t in range(T) if t % dk == m]
        tau = writers[-1]
        want[m] = v[0, tau, 0] * np.prod(alpha[tau + 1:, m])
    np.testing.assert_allclose(fs[0, 0], want, rtol=1e-13, atol=1e-15)

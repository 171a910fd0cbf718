"""Pins for the CPU fp64 oracle, each against something other than the oracle itself.

The pages fix the recurrence, the readout after the write, the two parents as
special cases, the overwrite / non-disturbance property and the
negative-eigenvalue extension; the tests below check the oracle against
those facts, a hand-worked exact example, closed forms, linearity, and an
independent (chunkwise, dense-inversion) formulation. A plausible mistake in
the oracle -- a dropped alpha in the residual, a transposed state, reading
before the write, a wrong decay, a sign error -- fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle.chunked import chunk_dense, chunk_fwd_dense

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(seed):
    return np.random.default_rng(seed)


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def make(seed, B=1, T=7, H=2, dk=5, dv=3, s0=True, beta_hi=1.0):
    r = rnd(seed)
    q = unit(r.standard_normal((B, T, H, dk)))
    k = unit(r.standard_normal((B, T, H, dk)))
    v = r.standard_normal((B, T, H, dv))
    g = -np.log1p(np.exp(r.standard_normal((B, T, H)) - 1.0))
    beta = r.uniform(0.05, beta_hi, (B, T, H))
    S0 = 0.3 * r.standard_normal((B, H, dk, dv)) if s0 else None
    return q, k, v, g, beta, S0


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# (d) hand-worked exact example -------------------------------------------------
def test_hand_worked_two_tokens():
    fx = json.load(open(os.path.join(GOLDEN, "hand_t2_dk2_dv3.json")))
    k = np.array(fx["k"], float)[None, :, None, :]
    q = np.array(fx["q"], float)[None, :, None, :]
    v = np.array(fx["v"], float)[None, :, None, :]
    g = np.log(np.array(fx["alpha"]))[None, :, None]
    beta = np.array(fx["beta"])[None, :, None]
    s0 = np.array(fx["initial_state"], float)[None, None]
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, s0)
    np.testing.assert_allclose(o[0, :, 0], np.array(fx["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(fs[0, 0], np.array(fx["final_state"]), rtol=0, atol=1e-14)
    # and the dense chunked form reproduces it too
    o2, fs2 = chunk_fwd_dense(q, k, v, g, beta, s0, chunk=2)
    np.testing.assert_allclose(o2[0, :, 0], np.array(fx["o"]), atol=1e-14)
    np.testing.assert_allclose(fs2[0, 0], np.array(fx["final_state"]), atol=1e-14)


# (a) beta = 0: pure decay, the Mamba2-parent limit -----------------------------
def test_beta_zero_is_pure_decay():
    q, k, v, g, beta, S0 = make(1, T=9)
    beta[:] = 0.0
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    Gam = np.cumsum(g, axis=1)                                   # [B,T,H]
    np.testing.assert_allclose(fs, np.exp(Gam[:, -1])[..., None, None] * S0, rtol=1e-13)
    # o_t = exp(Gamma_t) S_0 q_t, with S stored transposed: (S q)_i = sum_j st[j,i] q_j
    ref = np.exp(Gam)[..., None] * np.einsum("bhji,bthj->bthi", S0, q)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-14)


# (b) alpha = 1: ungated delta rule (DeltaNet parent) ---------------------------
def test_alpha_one_first_token_closed_form():
    q, k, v, g, beta, _ = make(2, T=1, H=3, dk=4, dv=6, s0=False)
    g[:] = 0.0
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, None)
    b = beta[0, 0]                                                # [H]
    # S_1 = beta v k^T, stored as state[j][i] = beta k_j v_i
    np.testing.assert_allclose(fs[0], b[:, None, None] * np.einsum("hj,hi->hji", k[0, 0], v[0, 0]),
                               rtol=1e-14)
    kq = np.einsum("hj,hj->h", k[0, 0], q[0, 0])
    np.testing.assert_allclose(o[0, 0], (b * kq)[:, None] * v[0, 0], rtol=1e-13)


def test_alpha_one_beta_zero_state_constant():
    q, k, v, g, beta, S0 = make(3, T=6)
    g[:] = 0.0
    beta[:] = 0.0
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    np.testing.assert_allclose(fs, S0, rtol=1e-15)
    np.testing.assert_allclose(o, np.einsum("bhji,bthj->bthi", S0, q), rtol=1e-13)


def test_alpha_one_matches_delta_rule_steps():
    # DeltaNet: S_t = S_{t-1} (I - beta k k^T) + beta v k^T, written as matrices
    q, k, v, g, beta, S0 = make(4, T=5, H=1, dk=3, dv=4)
    g[:] = 0.0
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    S = S0[0, 0].T.copy()
    for t in range(5):
        kt, vt, bt = k[0, t, 0], v[0, t, 0], beta[0, t, 0]
        S = S @ (np.eye(3) - bt * np.outer(kt, kt)) + bt * np.outer(vt, kt)
        np.testing.assert_allclose(o[0, t, 0], S @ q[0, t, 0], rtol=1e-12)
    np.testing.assert_allclose(fs[0, 0], S.T, rtol=1e-12)


# (c) overwrite, (f2) non-disturbance -------------------------------------------
def test_unit_key_beta_one_overwrites():
    q, k, v, g, beta, S0 = make(5, T=8, H=2, dk=6, dv=5)
    beta[:, -1] = 1.0                                             # last token: beta = 1
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    # S_T k_T = v_T exactly, whatever alpha and S_{T-1} are
    SkT = np.einsum("bhji,bhj->bhi", fs, k[:, -1])
    np.testing.assert_allclose(SkT, v[:, -1], rtol=1e-12, atol=1e-13)


def test_orthogonal_direction_only_decays():
    q, k, v, g, beta, S0 = make(6, T=1, H=2, dk=6, dv=4)
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    r = rnd(60)
    for h in range(2):
        kt = k[0, 0, h]
        kp = r.standard_normal(6)
        kp -= kp.dot(kt) * kt                                     # k' orthogonal to k_t
        lhs = fs[0, h].T @ kp
        rhs = np.exp(g[0, 0, h]) * (S0[0, h].T @ kp)
        np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-14)


# literal product form of the pages vs the oracle's expanded update -----------
def test_literal_product_form():
    q, k, v, g, beta, S0 = make(7, T=6, H=1, dk=4, dv=3, beta_hi=1.9)
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    S = S0[0, 0].T.copy()
    for t in range(6):
        kt, vt = k[0, t, 0], v[0, t, 0]
        a, b = np.exp(g[0, t, 0]), beta[0, t, 0]
        S = S @ (a * (np.eye(4) - b * np.outer(kt, kt))) + b * np.outer(vt, kt)
        np.testing.assert_allclose(o[0, t, 0], S @ q[0, t, 0], rtol=1e-12)
    np.testing.assert_allclose(fs[0, 0], S.T, rtol=1e-12)


# negative-eigenvalue extension: beta = 2 gives a reflection -------------------
def test_beta_two_reflects_the_key_direction():
    q, k, v, g, beta, S0 = make(8, T=1, H=1, dk=5, dv=3)
    g[:] = 0.0
    beta[:] = 2.0
    v[:] = 0.0
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    kt = k[0, 0, 0]
    np.testing.assert_allclose(fs[0, 0].T @ kt, -(S0[0, 0].T @ kt), rtol=1e-12)


# (f1) mutually orthogonal keys: gated linear attention closed form ------------
@pytest.mark.parametrize("with_s0", [False, True])
def test_orthogonal_keys_closed_form(with_s0):
    T, dk, dv = 6, 8, 3
    r = rnd(9)
    Qm, _ = np.linalg.qr(r.standard_normal((dk, dk)))
    k = Qm[:T][None, :, None, :]                                  # orthonormal keys
    q = unit(r.standard_normal((1, T, 1, dk)))
    v = r.standard_normal((1, T, 1, dv))
    g = -r.uniform(0.01, 0.5, (1, T, 1))
    beta = r.uniform(0.1, 1.0, (1, T, 1))
    S0 = 0.5 * r.standard_normal((1, 1, dk, dv)) if with_s0 else np.zeros((1, 1, dk, dv))
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    S0f = S0[0, 0].T
    gam = np.exp(np.cumsum(g[0, :, 0]))
    kk, qq, vv, bb = k[0, :, 0], q[0, :, 0], v[0, :, 0], beta[0, :, 0]
    u = bb[:, None] * (vv - gam[:, None] * (kk @ S0f.T))          # A = 0 => T = I
    for t in range(T):
        ref = gam[t] * S0f @ qq[t]
        for s in range(t + 1):
            ref = ref + gam[t] / gam[s] * kk[s].dot(qq[t]) * u[s]
        np.testing.assert_allclose(o[0, t, 0], ref, rtol=1e-12, atol=1e-14)


# linearity in (v, S_0) for fixed keys and gates --------------------------------
def test_linear_in_values_and_state():
    q, k, v1, g, beta, S1 = make(10, T=9)
    _, _, v2, _, _, S2 = make(11, T=9)
    o1, f1 = oracle.chunk_fwd(q, k, v1, g, beta, S1)
    o2, f2 = oracle.chunk_fwd(q, k, v2, g, beta, S2)
    o3, f3 = oracle.chunk_fwd(q, k, 2.0 * v1 - 3.0 * v2, g, beta, 2.0 * S1 - 3.0 * S2)
    np.testing.assert_allclose(o3, 2 * o1 - 3 * o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(f3, 2 * f1 - 3 * f2, rtol=1e-11, atol=1e-12)


# (e) dense chunkwise WY/UT form vs the token loop ------------------------------
@pytest.mark.parametrize("chunk", [1, 2, 4, 8, 64])
@pytest.mark.parametrize("T", [1, 7, 16, 21])
def test_dense_chunked_matches_token_loop(chunk, T):
    q, k, v, g, beta, S0 = make(12 + T, B=2, T=T, H=2, dk=8, dv=16, beta_hi=1.9)
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    o2, fs2 = chunk_fwd_dense(q, k, v, g, beta, S0, chunk=chunk)
    assert rel(o2, o) < 1e-12
    assert rel(fs2, fs) < 1e-12


def test_dense_chunked_intermediates_are_consistent():
    # T (I + A) = I; with A strictly lower the inverse is unit lower triangular
    q, k, v, g, beta, S0 = make(13, T=8, H=1, dk=4, dv=2)
    r = chunk_dense(k[0, :, 0], v[0, :, 0], q[0, :, 0], g[0, :, 0], beta[0, :, 0],
                    S0[0, 0].T)
    np.testing.assert_allclose(r["T"] @ (np.eye(8) + r["A"]), np.eye(8), atol=1e-13)
    np.testing.assert_allclose(np.triu(r["T"], 1), 0.0, atol=0)
    np.testing.assert_allclose(np.diag(r["T"]), 1.0, atol=1e-15)


# varlen = separate calls; split sequence = one call ----------------------------
def test_varlen_equals_separate_sequences():
    lens = [3, 1, 6, 2]
    q, k, v, g, beta, _ = make(14, B=1, T=sum(lens), H=2, dk=4, dv=5)
    S0 = 0.2 * rnd(15).standard_normal((len(lens), 2, 4, 5))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0, cu)
    for n in range(len(lens)):
        sl = slice(cu[n], cu[n + 1])
        on, fn = oracle.chunk_fwd(q[:, sl], k[:, sl], v[:, sl], g[:, sl], beta[:, sl],
                                  S0[n:n + 1])
        np.testing.assert_allclose(o[:, sl], on, rtol=1e-14)
        np.testing.assert_allclose(fs[n], fn[0], rtol=1e-14)


def test_split_sequence_hands_over_state():
    q, k, v, g, beta, S0 = make(16, B=2, T=11, H=2)
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    oa, fa = oracle.chunk_fwd(q[:, :4], k[:, :4], v[:, :4], g[:, :4], beta[:, :4], S0)
    ob, fb = oracle.chunk_fwd(q[:, 4:], k[:, 4:], v[:, 4:], g[:, 4:], beta[:, 4:], fa)
    np.testing.assert_allclose(np.concatenate([oa, ob], 1), o, rtol=1e-13)
    np.testing.assert_allclose(fb, fs, rtol=1e-13)


def test_decode_step_is_one_token():
    q, k, v, g, beta, S0 = make(17, B=3, T=1, H=2, dk=4, dv=6)
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    od, sd = oracle.decode_step(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], S0)
    np.testing.assert_allclose(od, o[:, 0], rtol=1e-15)
    np.testing.assert_allclose(sd, fs, rtol=1e-15)


def test_empty_sequence_keeps_state():
    q, k, v, g, beta, S0 = make(18, B=1, T=0, H=2)
    o, fs = oracle.chunk_fwd(q, k, v, g, beta, S0)
    assert o.shape == (1, 0, 2, 3)
    np.testing.assert_array_equal(fs, S0)


def test_rejects_bad_cu_seqlens():
    q, k, v, g, beta, _ = make(19, B=1, T=5)
    with pytest.raises(ValueError):
        oracle.chunk_fwd(q, k, v, g, beta, None, np.array([0, 3, 2, 5], np.int32))

"""Pins for the backward-pass oracle (``oracle.chunk_bwd``), each against
something other than that function.

The pages describe the chunkwise algorithm as a training algorithm but give
no gradients (phantomic12 page, mechanism paragraph); they are derived by
reverse-mode differentiation of the recurrence. These tests check them
against central finite differences of the forward oracle (pinned on its
own), against two homogeneity identities that hold exactly (o and the final
state are jointly linear in (V, S_0); o is linear in each q_t), against the
closed form of the pure-decay case beta = 0, and against splitting a packed
batch into separate sequences.
"""
import numpy as np
import pytest

import oracle


def make(seed, B=1, T=7, H=1, dk=3, dv=2, s0=True, varlen=None):
    r = np.random.default_rng(seed)
    if varlen is not None:
        B, T = 1, int(sum(varlen))
    q = 0.5 * r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, dv))
    g = -np.log1p(np.exp(r.standard_normal((B, T, H)) - 1.0))
    beta = r.uniform(0.05, 1.0, (B, T, H))
    N = len(varlen) if varlen is not None else B
    S0 = 0.5 * r.standard_normal((N, H, dk, dv)) if s0 else None
    d_o = r.standard_normal((B, T, H, dv))
    dsN = r.standard_normal((N, H, dk, dv))
    cu = None if varlen is None else np.concatenate([[0], np.cumsum(varlen)]).astype(np.int32)
    return dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0, d_o=d_o, dsN=dsN, cu=cu)


def loss(a, **over):
    b = dict(a, **over)
    o, fs = oracle.chunk_fwd(b["q"], b["k"], b["v"], b["g"], b["beta"], b["S0"], b["cu"],
                             nthreads=1)
    return float((o * b["d_o"]).sum() + (fs * b["dsN"]).sum())


def grads(a):
    return oracle.chunk_bwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["d_o"], a["S0"],
                            a["cu"], a["dsN"], nthreads=1)


NAMES = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "beta": "dbeta", "S0": "d_initial_state"}


def central_differences(a, name, eps=1e-6):
    x = a[name]
    fd = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += eps
        xm[idx] -= eps
        fd[idx] = (loss(a, **{name: xp}) - loss(a, **{name: xm})) / (2 * eps)
    return fd


@pytest.mark.parametrize("case", ["plain", "no_s0", "two_blocks", "varlen"])
def test_bwd_matches_central_differences(case):
    if case == "plain":
        a = make(1)
    elif case == "no_s0":
        a = make(2, s0=False)
    elif case == "two_blocks":   # crosses the oracle's 64-token recompute boundary
        a = make(3, T=70, dk=2, dv=2)
    else:
        a = make(4, varlen=[3, 0, 5])
    gr = grads(a)
    for name, gname in NAMES.items():
        if a[name] is None:
            continue
        fd = central_differences(a, name)
        err = np.max(np.abs(fd - gr[gname]))
        assert err <= 1e-7 * max(1.0, np.max(np.abs(fd))), f"{gname}: {err:.2e}"


def test_bwd_homogeneity_identities():
    # o and the final state are jointly linear in (V, S_0): by Euler's theorem
    # sum(v * dv) + sum(S_0 * dS_0) = L. o_t is linear in q_t and the final
    # state does not depend on q: sum(q * dq) = sum(d_o * o).
    a = make(5, T=40, H=2, dk=4, dv=3)
    gr = grads(a)
    L = loss(a)
    lhs = float((a["v"] * gr["dv"]).sum() + (a["S0"] * gr["d_initial_state"]).sum())
    assert abs(lhs - L) <= 1e-12 * max(1.0, abs(L))
    o, _ = oracle.chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"])
    assert abs(float((a["q"] * gr["dq"]).sum()) - float((o * a["d_o"]).sum())) <= 1e-12 * max(
        1.0, abs(float((o * a["d_o"]).sum())))


def test_bwd_beta_zero_closed_form():
    # beta = 0: S_t = gamma_t S_0, o_t = gamma_t S_0 q_t, S_T = gamma_T S_0, so
    # dq_t = gamma_t S_0^T do_t, dv = dk = 0, dS_0 = sum_t gamma_t do_t q_t^T + gamma_T dS_T,
    # dg_s = sum_{t >= s} gamma_t do_t . (S_0 q_t) + gamma_T <dS_T, S_0>.
    a = make(6, T=9, dk=3, dv=4)
    a["beta"][:] = 0.0
    gr = grads(a)
    S0 = a["S0"][0, 0].T                          # formula orientation d_v x d_k
    gam = np.exp(np.cumsum(a["g"][0, :, 0]))
    q, do, dsN = a["q"][0, :, 0], a["d_o"][0, :, 0], a["dsN"][0, 0].T
    np.testing.assert_allclose(gr["dq"][0, :, 0], gam[:, None] * (do @ S0), rtol=1e-12,
                               atol=1e-14)
    assert np.max(np.abs(gr["dv"])) == 0.0 and np.max(np.abs(gr["dk"])) == 0.0
    want_ds0 = sum(gam[t] * np.outer(do[t], q[t]) for t in range(9)) + gam[-1] * dsN
    np.testing.assert_allclose(gr["d_initial_state"][0, 0], want_ds0.T, rtol=1e-12, atol=1e-14)
    per_t = gam * np.einsum("ti,ij,tj->t", do, S0, q)
    want_dg = np.cumsum(per_t[::-1])[::-1] + gam[-1] * float((dsN * S0).sum())
    np.testing.assert_allclose(gr["dg"][0, :, 0], want_dg, rtol=1e-12, atol=1e-14)


def test_bwd_varlen_equals_separate_sequences():
    lens = [4, 0, 6, 2]
    a = make(7, varlen=lens, H=2)
    gr = grads(a)
    cu = a["cu"]
    for n in range(len(lens)):
        s, e = cu[n], cu[n + 1]
        b = dict(q=a["q"][:, s:e], k=a["k"][:, s:e], v=a["v"][:, s:e], g=a["g"][:, s:e],
                 beta=a["beta"][:, s:e], S0=a["S0"][n:n + 1], d_o=a["d_o"][:, s:e],
                 dsN=a["dsN"][n:n + 1], cu=None)
        gn = grads(b)
        for key in ("dq", "dk", "dv", "dg", "dbeta"):
            np.testing.assert_allclose(gr[key][:, s:e], gn[key], rtol=0, atol=1e-14)
        np.testing.assert_allclose(gr["d_initial_state"][n], gn["d_initial_state"][0], rtol=0,
                                   atol=1e-14)


def test_bwd_is_causal():
    # a loss on the outputs of tokens < t_cut only: no gradient reaches the
    # inputs of later tokens (exact zeros, not small numbers)
    a = make(8, T=12, H=2, dk=3, dv=4)
    t_cut = 7
    a["d_o"][:, t_cut:] = 0.0
    a["dsN"][:] = 0.0
    gr = grads(a)
    for key in ("dk", "dv", "dg", "dbeta", "dq"):
        assert np.max(np.abs(gr[key][:, t_cut:])) == 0.0, key
    assert np.max(np.abs(gr["dv"][:, :t_cut])) > 0.0

"""The chunkwise gradient formulas that the tensor-core backward kernels
compute, restated in fp64 numpy, against the oracle's token-level
reverse-mode gradients (``oracle.chunk_bwd``).

The pages give no gradients for the chunkwise algorithm ("Gated Delta
Networks", phantomic12 page, mechanism paragraph: a training algorithm); the
kernels differentiate the chunk equations instead of the token recurrence.
This test pins that derivation on the CPU: every gradient (dq, dk, dv, dg,
dbeta, d_initial_state) must agree with the token-level oracle to rounding,
for chunk sizes that leave a ragged tail, d_k != d_v, beta up to 2 and
rows with beta = 0. The restatement is test code; it shares nothing with the
CUDA kernels (which run the same steps on bf16 tiles)."""
import numpy as np
import pytest

import oracle
from oracle.chunked import chunk_dense


def chunkwise_bwd(q, k, v, g, b, do, s0, dsN, C):
    """One (sequence, head): q, k [T, d_k], v, do [T, d_v], g, b [T],
    s0, dsN [d_v, d_k] in the formula orientation."""
    T = q.shape[0]
    nc = (T + C - 1) // C
    S = s0.copy()
    Sc, F = [], []
    for c in range(nc):
        sl = slice(c * C, min(T, (c + 1) * C))
        f = chunk_dense(k[sl], v[sl], q[sl], g[sl], b[sl], S)
        Sc.append(S.copy())
        F.append(f)
        S = f["S_next"]
    # reverse chain over the chunks: dS_c = gamma_last G' - dX^T W + (gamma dO)^T Q
    G, Gp = dsN.copy(), [None] * nc
    for c in reversed(range(nc)):
        sl = slice(c * C, min(T, (c + 1) * C))
        f = F[c]
        gam = np.exp(f["Gamma"])
        D = np.exp(f["Gamma"][-1] - f["Gamma"])
        Gp[c] = G.copy()
        dX = f["P"].T @ do[sl] + (D[:, None] * k[sl]) @ G.T
        G = gam[-1] * G - dX.T @ f["W"] + (gam[:, None] * do[sl]).T @ q[sl]
    out = {key: np.zeros_like(a) for key, a in (("dq", q), ("dk", k), ("dv", v))}
    out["dg"], out["dbeta"], out["ds0"] = np.zeros(T), np.zeros(T), G
    for c in range(nc):
        sl = slice(c * C, min(T, (c + 1) * C))
        f, S, Gq = F[c], Sc[c], Gp[c]
        Q, K, V, dO = q[sl], k[sl], v[sl], do[sl]
        L = Q.shape[0]
        Gam = f["Gamma"]
        gam, D = np.exp(Gam), np.exp(Gam[-1] - Gam)
        E = np.exp(Gam[:, None] - Gam[None, :])
        strict, incl = np.tril(np.ones((L, L)), -1), np.tril(np.ones((L, L)), 0)
        TB = f["T"] * b[sl][None, :]
        X = TB @ V - f["W"] @ S.T
        DKG = (D[:, None] * K) @ Gq.T
        dX = f["P"].T @ dO + DKG
        dV = TB.T @ dX
        Lm = (K @ K.T) * E * strict
        dY = dX - Lm.T @ dV
        e = V - gam[:, None] * (K @ S.T) - Lm @ X
        dP = dO @ X.T
        dPt = dP * E * incl
        Rp = dV @ X.T
        R = -Rp * E * strict
        dOS, dVS = dO @ S, dV @ S
        out["dq"][sl] = gam[:, None] * dOS + dPt @ K
        out["dk"][sl] = (dPt.T @ Q + D[:, None] * (X @ Gq) - gam[:, None] * dVS + R @ K
                         + R.T @ K)
        out["dv"][sl] = dV
        out["dbeta"][sl] = np.sum(dY * e, axis=1)
        Pf, Af = dP * f["P"], -Rp * Lm
        delta = np.sum(X * DKG, axis=1)
        dGam = (gam * np.sum(Q * dOS, 1) - gam * np.sum(K * dVS, 1) + Pf.sum(1) - Pf.sum(0)
                + Af.sum(1) - Af.sum(0) - delta)
        dGam[-1] += delta.sum() + gam[-1] * np.sum(Gq * S)
        out["dg"][sl] = np.cumsum(dGam[::-1])[::-1]
    return out


@pytest.mark.parametrize("T,dk,dv,C", [(1, 8, 6, 4), (7, 8, 6, 4), (64, 16, 12, 16),
                                        (150, 16, 12, 16), (200, 32, 24, 64)])
def test_chunkwise_gradients_equal_the_token_level_oracle(T, dk, dv, C):
    rng = np.random.default_rng(T + dk)
    unit = lambda a: a / np.linalg.norm(a, axis=1, keepdims=True)
    q, k = unit(rng.standard_normal((T, dk))), unit(rng.standard_normal((T, dk)))
    v, do = rng.standard_normal((T, dv)), rng.standard_normal((T, dv))
    g = -np.log1p(np.exp(rng.standard_normal(T) - 2.0))
    b = 2.0 / (1.0 + np.exp(-rng.standard_normal(T)))          # beta in (0, 2)
    b[::5] = 0.0                                                # and some beta = 0 rows
    s0, dsN = 0.1 * rng.standard_normal((dv, dk)), 0.1 * rng.standard_normal((dv, dk))
    got = chunkwise_bwd(q, k, v, g, b, do, s0, dsN, C)
    lift = lambda a: a[None, :, None]
    ref = oracle.chunk_bwd(lift(q), lift(k), lift(v), lift(g), lift(b), lift(do),
                           s0.T[None, None], None, dsN.T[None, None], nthreads=1)
    for key in ("dq", "dk", "dv", "dg", "dbeta"):
        np.testing.assert_allclose(got[key], ref[key][0, :, 0], rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(got["ds0"].T, ref["d_initial_state"][0, 0], rtol=1e-10,
                               atol=1e-11)

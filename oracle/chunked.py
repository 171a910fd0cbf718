"""Dense chunkwise (WY / UT-transform) form of the gated delta rule, in numpy fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages name the parallel algorithm -- a WY representation / UT transform
applied chunkwise, extended to carry the decay gate (phantomic12
"gated-deltanet" page, mechanism paragraph; dmarx anthology LIT-137,
"Standing in the anthology"; SOTA-135, "Source") -- but print none of its
equations. They follow from unrolling the recurrence over one chunk that
starts from state S_0 (rows r, s in [0, C) of the chunk):

    Gamma_r = sum_{s <= r} g_s,   gamma_r = exp(Gamma_r)
    u_r     = beta_r (v_r - alpha_r S_{r-1} k_r)            (pseudo-values)
    S_r     = gamma_r S_0 + sum_{s <= r} (gamma_r / gamma_s) u_s k_s^T

Substituting S_{r-1} into u_r gives a unit lower-triangular system

    (I + A) u = diag(beta) V - diag(beta gamma) K S_0^T,
    A_rs = beta_r exp(Gamma_r - Gamma_s) (k_r . k_s)  for s < r, else 0,

so with the UT transform T = (I + A)^{-1}:

    W = T diag(beta gamma) K,   U = T diag(beta) V,   V_new = U - W S_0^T
    O = diag(gamma) Q S_0^T + (Q K^T (.) M) V_new,  M_rs = exp(Gamma_r - Gamma_s), s <= r
    S_C = gamma_{C-1} S_0 + V_new^T diag(exp(Gamma_{C-1} - Gamma)) K

The readout mask includes the diagonal because o_t reads the state after
the write at t (portpowered "Gated DeltaNet" page, "How It Works"). T is
obtained by a dense solve (a library primitive), not by the blocked
substitution the kernels use.
"""
from __future__ import annotations

import numpy as np


def chunk_dense(Kc, Vc, Qc, gc, bc, S0):
    """Apply the chunk equations above to one chunk.

    Kc, Qc: [L, d_k]; Vc: [L, d_v]; gc, bc: [L]; S0: [d_v, d_k] (formula
    orientation). L may be shorter than the chunk size (a ragged tail).
    Returns dict with Gamma, A, T, W, U, V_new, P (= QK^T (.) M), O, S_next.
    """
    L = Kc.shape[0]
    Gam = np.cumsum(gc)
    gam = np.exp(Gam)
    diff = Gam[:, None] - Gam[None, :]
    lower = np.tril(np.ones((L, L), dtype=bool), -1)
    incl = np.tril(np.ones((L, L), dtype=bool), 0)
    decay = np.where(incl, np.exp(np.where(incl, diff, 0.0)), 0.0)
    A = np.where(lower, bc[:, None] * decay * (Kc @ Kc.T), 0.0)
    T = np.linalg.solve(np.eye(L) + A, np.eye(L))
    W = T @ ((bc * gam)[:, None] * Kc)
    U = T @ (bc[:, None] * Vc)
    Vnew = U - W @ S0.T
    P = (Qc @ Kc.T) * decay
    O = gam[:, None] * (Qc @ S0.T) + P @ Vnew
    D = np.exp(Gam[-1] - Gam) if L else np.zeros(0)
    S_next = (gam[-1] if L else 1.0) * S0 + Vnew.T @ (D[:, None] * Kc)
    return dict(Gamma=Gam, A=A, T=T, W=W, U=U, V_new=Vnew, P=P, O=O, S_next=S_next)


def chunk_fwd_dense(q, k, v, g, beta, initial_state=None, cu_seqlens=None, chunk=64,
                    keep=False):
    """Whole-sequence forward by chunks of ``chunk`` tokens (fp64).

    Same argument layout as ``oracle.chunk_fwd``. Chunks start at each
    sequence's first token; the last chunk of a sequence may be partial.
    With ``keep=True`` also returns the per-chunk intermediates as a list of
    dicts keyed by (seq, head, chunk index).
    """
    q, k, v, g, beta = (np.asarray(a, dtype=np.float64) for a in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        cu = [int(x) for x in np.asarray(cu_seqlens)]
        spans = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    else:
        spans = [(b, 0, T) for b in range(B)]
    N = len(spans)
    o = np.zeros((B, T, H, dv))
    fs = np.zeros((N, H, dk, dv))
    inter = {}
    for n, (b, t0, t1) in enumerate(spans):
        for h in range(H):
            S = (np.zeros((dv, dk)) if initial_state is None
                 else np.asarray(initial_state, dtype=np.float64)[n, h].T.copy())
            for ci, c0 in enumerate(range(t0, t1, chunk)):
                c1 = min(c0 + chunk, t1)
                r = chunk_dense(k[b, c0:c1, h], v[b, c0:c1, h], q[b, c0:c1, h],
                                g[b, c0:c1, h], beta[b, c0:c1, h], S)
                o[b, c0:c1, h] = r["O"]
                if keep:
                    r["S0"] = S
                    inter[(n, h, ci)] = r
                S = r["S_next"]
            fs[n, h] = S.T
    if keep:
        return o, fs, inter
    return o, fs

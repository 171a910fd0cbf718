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


def kda_chunk_dense(Kc, Vc, Qc, Gc, bc, S0):
    """The chunk equations for the channel-wise gate (g = log alpha per d_k
    channel; the Kimi Delta Attention variant, named on the dmarx anthology
    LIT-137 page, "Standing in the anthology", and SOTA-135, "Sequence").

    With S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    unrolling one chunk from S_0 gives, per channel j, Gamma_rj = sum_{s<=r} g_sj
    and

        S_r = S_0 diag(exp(Gamma_r)) + sum_{s<=r} u_s (k_s (.) exp(Gamma_r - Gamma_s))^T
        u_r = beta_r (v_r - S_{r-1} diag(alpha_r) k_r)

    so the decay moves inside the dot products:

        A_rs = beta_r sum_j k_rj k_sj exp(Gamma_rj - Gamma_sj)   (s < r)
        T = (I + A)^-1,  W = T diag(beta) (K (.) exp(Gamma)),  U = T diag(beta) V
        V_new = U - W S_0^T
        P_rs = sum_j q_rj k_sj exp(Gamma_rj - Gamma_sj)          (s <= r)
        O = (Q (.) exp(Gamma)) S_0^T + P V_new
        S_C = S_0 diag(exp(Gamma_last)) + V_new^T (K (.) exp(Gamma_last - Gamma))

    Gc: [L, d_k]; other arguments as in ``chunk_dense``. Every exponent above
    is a difference of cumulative sums taken over the tokens in between, as
    written (no rescaling).
    """
    L = Kc.shape[0]
    Gam = np.cumsum(Gc, axis=0)                            # [L, d_k]
    incl = np.tril(np.ones((L, L), dtype=bool), 0)
    lower = np.tril(np.ones((L, L), dtype=bool), -1)
    diff = Gam[:, None, :] - Gam[None, :, :]               # [r, s, j]
    E = np.where(incl[:, :, None], np.exp(np.where(incl[:, :, None], diff, 0.0)), 0.0)
    KK = np.einsum("rj,sj,rsj->rs", Kc, Kc, E)
    A = np.where(lower, bc[:, None] * KK, 0.0)
    T = np.linalg.solve(np.eye(L) + A, np.eye(L))
    W = T @ (bc[:, None] * (Kc * np.exp(Gam)))
    U = T @ (bc[:, None] * Vc)
    Vnew = U - W @ S0.T
    P = np.einsum("rj,sj,rsj->rs", Qc, Kc, E)
    O = (Qc * np.exp(Gam)) @ S0.T + P @ Vnew
    if L:
        S_next = S0 * np.exp(Gam[-1])[None, :] + Vnew.T @ (Kc * np.exp(Gam[-1][None, :] - Gam))
    else:
        S_next = S0.copy()
    return dict(Gamma=Gam, A=A, T=T, W=W, U=U, V_new=Vnew, P=P, O=O, S_next=S_next)


def chunk_fwd_dense(q, k, v, g, beta, initial_state=None, cu_seqlens=None, chunk=64,
                    keep=False, channel_gate=False):
    """Whole-sequence forward by chunks of ``chunk`` tokens (fp64).

    Same argument layout as ``oracle.chunk_fwd`` (``oracle.kda_chunk_fwd``
    with ``channel_gate=True``: g is [B,T,H,d_k]). Chunks start at each
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
                step = kda_chunk_dense if channel_gate else chunk_dense
                r = step(k[b, c0:c1, h], v[b, c0:c1, h], q[b, c0:c1, h],
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


def kda_chunk_fwd_dense(q, k, v, g, beta, initial_state=None, cu_seqlens=None, chunk=64,
                        keep=False):
    """``chunk_fwd_dense`` for the channel-wise gate (g: [B,T,H,d_k])."""
    return chunk_fwd_dense(q, k, v, g, beta, initial_state, cu_seqlens, chunk, keep,
                           channel_gate=True)

"""fp64 numpy statement of the chunkwise (WY / UT-transform) form of KDA.

This is the algebra the CUDA chunk kernels implement, written plainly so a test
can prove it equals the token recurrence to fp64 rounding. It is a check of the
derivation, not the oracle (the oracle is the token recurrence).

Derivation (Kimi Linear summary, section 3.1 "Hardware-Efficient Chunkwise
Algorithm" describes it in prose; the steps below are derived from the KDA
recurrence of section 3). For one chunk of C rows entering with state S0, let
G_r = sum_{j<=r} log alpha_j (per channel, inclusive) and gamma_r = exp(G_r):

    A_{ri} = beta_r sum_c k_rc exp(G_rc - G_ic) k_ic      (i < r, strictly lower)
    P_{ri} =        sum_c q_rc exp(G_rc - G_ic) k_ic      (i <= r, lower incl. diagonal)
    T      = (I + A)^{-1}                                 (unit lower; forward substitution)
    W      = T diag(beta) (K * gamma)                     U = T diag(beta) V
    Delta  = U - W S0                                     (rows = effective writes delta_r)
    O      = (Q * gamma) S0 + P Delta
    S_C    = Diag(exp(G_C)) S0 + (K * exp(G_C - G))^T Delta

Each chunk starts from the previous chunk's final state; a ragged last chunk
simply has fewer rows.
"""

from __future__ import annotations

import numpy as np


def forward_substitution_inverse(A):
    """T = (I + A)^{-1} for strictly lower-triangular A, solved row by row."""
    C = A.shape[0]
    T = np.zeros_like(A)
    for r in range(C):
        T[r, r] = 1.0
        for i in range(r):
            # row r of (I + A) T = I:  T[r, :] = e_r - sum_{m<r} A[r, m] T[m, :]
            T[r, :] -= A[r, i] * T[i, :]
    return T


def chunk_forward(q, k, v, beta, log_alpha, S0=None, chunk: int = 64):
    """Single head. q, k, log_alpha [T, dk]; v [T, dv]; beta [T]. Returns (o, S_T)."""
    q, k, v, beta, la = (np.asarray(x, dtype=np.float64) for x in (q, k, v, beta, log_alpha))
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        Q, K, V, B, L = q[t0:t1], k[t0:t1], v[t0:t1], beta[t0:t1], la[t0:t1]
        C = t1 - t0
        G = np.cumsum(L, axis=0)                       # [C, dk]
        diff = G[:, None, :] - G[None, :, :]           # G_r - G_i, [C, C, dk]
        mask_strict = np.tril(np.ones((C, C)), -1)
        mask_incl = np.tril(np.ones((C, C)), 0)
        E = np.exp(np.where(mask_incl[:, :, None] > 0, diff, 0.0))
        A = B[:, None] * np.einsum("rc,ric,ic->ri", K, E, K) * mask_strict
        P = np.einsum("rc,ric,ic->ri", Q, E, K) * mask_incl
        Tm = forward_substitution_inverse(A)
        gamma = np.exp(G)
        W = Tm @ (B[:, None] * (K * gamma))
        U = Tm @ (B[:, None] * V)
        Delta = U - W @ S
        o[t0:t1] = (Q * gamma) @ S + P @ Delta
        gC = G[-1]
        S = np.exp(gC)[:, None] * S + (K * np.exp(gC[None, :] - G)).T @ Delta
    return o, S


def dplr_chunked(q, k, v, a, b, log_alpha, S0, C=64):
    """General DPLR, S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T, by chunks (fp64,
    one head), derived from the recurrence: within a chunk with inclusive cumulative log
    decay G (G_{-1} = 0) and correction rows u_r = b_r^T S_{r-1},
        S_r = Diag(e^{G_r}) S_0 + sum_{i<=r} Diag(e^{G_r - G_i}) (k_i v_i^T - a_i u_i^T),
    so with the decayed Grams (i < r)  Mbk_ri = b_r . (e^{G_{r-1} - G_i} k_i),
    Mba_ri = b_r . (e^{G_{r-1} - G_i} a_i) and (i <= r)  Mqk_ri = q_r . (e^{G_r - G_i} k_i),
    Mqa_ri = q_r . (e^{G_r - G_i} a_i):
        (I + Mba) U = (B * e^{G_prev}) S_0 + Mbk V
        O = (Q * e^G) S_0 + Mqk V - Mqa U
        S_C = Diag(e^{G_C}) S_0 + (K * e^{G_C - G})^T V - (A * e^{G_C - G})^T U.
    Four decayed Grams where KDA's tied factors need two."""
    T, dk = q.shape
    S = np.array(S0, dtype=np.float64)
    o = np.zeros((T, v.shape[1]))
    for t0 in range(0, T, C):
        sl = slice(t0, min(T, t0 + C))
        Q, K, V, A, B = q[sl], k[sl], v[sl], a[sl], b[sl]
        G = np.cumsum(log_alpha[sl], axis=0)
        Gp = np.vstack([np.zeros((1, dk)), G[:-1]])
        L = Q.shape[0]
        Mbk = np.zeros((L, L)); Mba = np.zeros((L, L)); Mqk = np.zeros((L, L)); Mqa = np.zeros((L, L))
        for r in range(L):
            for i in range(r + 1):
                ec = np.exp(G[r] - G[i])
                Mqk[r, i] = Q[r] @ (ec * K[i])
                Mqa[r, i] = Q[r] @ (ec * A[i])
                if i < r:
                    ep = np.exp(Gp[r] - G[i])
                    Mbk[r, i] = B[r] @ (ep * K[i])
                    Mba[r, i] = B[r] @ (ep * A[i])
        U = np.linalg.solve(np.eye(L) + Mba, (B * np.exp(Gp)) @ S + Mbk @ V)
        o[sl] = (Q * np.exp(G)) @ S + Mqk @ V - Mqa @ U
        F = np.exp(G[-1] - G)
        S = np.exp(G[-1])[:, None] * S + (K * F).T @ V - (A * F).T @ U
    return o, S

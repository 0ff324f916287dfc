"""The chunk form in the end-of-chunk factorisation the tensor-core kernel uses, with a
rounding hook at every matrix-product operand (fp64 arithmetic in between).

Kimi Linear summary, section 3.1 "Hardware-Efficient Chunkwise Algorithm", gives the
chunkwise WY/UT form; the factorisation below is this repository's way of evaluating it
with one Gram product per chunk. For one chunk with inclusive cumulative log-decay G
(rows r) and last row G_C:

    E = exp(G - G_C) >= 1,  F = exp(G_C - G) <= 1,  so exp(G_r - G_i) = E_r F_i
    Rk = K*E, Rq = Q*E, Ck = K*F,  S'' = Diag(exp(G_C)) S
    A = beta (Rk Ck^T) strictly lower,  P = Rq Ck^T lower with the diagonal
    Tb = (I + A)^{-1} Diag(beta),  W' = Tb Rk,  U = Tb V
    Delta = U - W' S'',  O = Rq S'' + P Delta,  S <- S'' + Ck^T Delta

Every operand of a product passes through a rounding function chosen by the caller
(identity: the exact form; bf16 or tf32: a tensor-core operand), and every product is
rounded to fp32 as an fp32 accumulator would hold it. Test infrastructure only.
"""

from __future__ import annotations

import numpy as np


def as_f32(x):
    return np.asarray(x, np.float32).astype(np.float64)


def exact(x):
    return np.asarray(x, np.float64)


def round_bf16(x):
    """Round to the nearest bf16 (ties to even), through the fp32 bit pattern."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def round_tf32(x):
    """Round to the nearest tf32 (10 explicit mantissa bits, ties to even)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0xFFF + ((u >> 13) & 1)) & 0xFFFFE000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def _unit_lower_inverse(A):
    C = A.shape[0]
    T = np.zeros_like(A)
    for r in range(C):
        T[r, r] = 1.0
        for i in range(r):
            T[r, :] -= A[r, i] * T[i, :]
    return T


def chunk_forward_rounded(q, k, v, beta, log_alpha, S0, tiles=exact, t_beta=exact,
                          state=exact, left=exact, update=exact, acc=exact, out=exact,
                          chunk: int = 64):
    """Single head. q, k, log_alpha [T, dk]; v [T, dv]; beta [T]; S0 [dk, dv].

    Rounding hooks: `tiles` for Rk, Rq, Ck and V as Gram/W'/U operands, `t_beta` for Tb,
    `state` for S'' as an operand, `left` for [Rq; -W'] against S'', `update` for Ck and
    Delta in the state update and P Delta, `acc` for every accumulator, `out` for o.
    Returns (o [T, dv], S_T [dk, dv]).
    """
    q, k, v, beta, la = (np.asarray(x, np.float64) for x in (q, k, v, beta, log_alpha))
    S = acc(np.array(S0, np.float64))
    o = np.zeros((q.shape[0], v.shape[1]))
    for t0 in range(0, q.shape[0], chunk):
        t1 = min(q.shape[0], t0 + chunk)
        Q, K, V, L, B = q[t0:t1], k[t0:t1], v[t0:t1], la[t0:t1], beta[t0:t1]
        C = t1 - t0
        G = np.cumsum(L, axis=0)
        GC = G[-1]
        E, F = np.exp(G - GC), np.exp(GC - G)
        Rk, Rq, Ck = tiles(K * E), tiles(Q * E), tiles(K * F)
        A = acc(B[:, None] * (Rk @ Ck.T)) * np.tril(np.ones((C, C)), -1)
        P = acc(Rq @ Ck.T) * np.tril(np.ones((C, C)), 0)
        Tb = t_beta(_unit_lower_inverse(A) * B[None, :])
        Wp = acc(Tb @ Rk)
        U = acc(Tb @ tiles(V))
        Spp = acc(np.exp(GC)[:, None] * S)
        Sop = state(Spp)
        D = acc(U - left(Wp) @ Sop)
        Dop = update(D)
        o[t0:t1] = out(acc(left(Rq) @ Sop + update(P) @ Dop))
        S = acc(Spp + update(Ck).T @ Dop)
    return o, S

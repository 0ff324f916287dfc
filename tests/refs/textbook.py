"""Independently written textbook recurrences used to pin the KDA oracle.

Each function here is written from its own textbook definition, not from the
KDA oracle, in plain fp64 numpy on a single head. Sources (Kimi Linear
summaries):

* linear attention: S_t = S_{t-1} + k_t v_t^T, o_t = S_t^T q_t
  ("Rationalist Deep-Dive", section 2.1 "The Fast-Weight Lens");
* DeltaNet as one gradient step of size beta_t on L_t(S) = 1/2 ||S^T k_t - v_t||^2
  (same page, section 2.2 "DeltaNet: Attention as Gradient Descent"); coded here
  as the gradient step itself, S <- S - beta * k (S^T k - v)^T;
* Gated DeltaNet with a scalar forget gate: S_t = a_t (I - beta k k^T) S_{t-1} + beta k v^T
  (same page, section 2.3, and "KDA: Splitting the Decay Across Channels");
* GLA, a per-channel gate with an additive write: S_t = Diag(alpha_t) S_{t-1} + k_t v_t^T
  ("KDA: Splitting the Decay Across Channels", the remark that this gate already
  appeared in GLA);
* the unrolled (parallel) form, o_t = q_t^T (prod_{j=i+1..t} A_j) beta_i k_i v_i^T summed
  over i <= t plus the carried initial state, with the explicit d_k x d_k transition
  A_j = (I - beta_j k_j k_j^T) Diag(alpha_j) ("Rationalist Deep-Dive" section 3.3 and the
  summary's section 6.1, with beta_i restored on each write as the KDA recurrence in
  section 3 states).
"""

from __future__ import annotations

import numpy as np


def linear_attention(q, k, v, S0=None):
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    for t in range(T):
        S = S + np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def deltanet_gradient_step(q, k, v, beta, S0=None):
    """DeltaNet written as SGD on the per-step reconstruction loss."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    for t in range(T):
        grad = np.outer(k[t], S.T @ k[t] - v[t])     # dL/dS for L = 1/2 ||S^T k - v||^2
        S = S - beta[t] * grad
        o[t] = S.T @ q[t]
    return o, S


def gated_deltanet_scalar(q, k, v, beta, a, S0=None):
    """Gated DeltaNet with one scalar gate a_t per step."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    eye = np.eye(dk)
    for t in range(T):
        S = a[t] * (eye - beta[t] * np.outer(k[t], k[t])) @ S + beta[t] * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def gla(q, k, v, alpha, S0=None):
    """Gated linear attention: per-channel decay, additive write, no delta rule."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    for t in range(T):
        S = alpha[t][:, None] * S + np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def kda_unrolled(q, k, v, beta, alpha, S0=None):
    """Brute-force parallel form with explicit transition products (tiny T only).

    o_t = q_t^T [ (A_t ... A_1) S0 + sum_{i<=t} (A_t ... A_{i+1}) beta_i k_i v_i^T ].
    """
    T, dk = q.shape
    dv = v.shape[1]
    S0 = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    eye = np.eye(dk)
    A = [(eye - beta[j] * np.outer(k[j], k[j])) @ np.diag(alpha[j]) for j in range(T)]

    def prod(lo, hi):  # A_hi ... A_lo (inclusive), identity when empty
        P = eye.copy()
        for j in range(lo, hi + 1):
            P = A[j] @ P
        return P

    o = np.zeros((T, dv))
    for t in range(T):
        M = prod(0, t) @ S0
        for i in range(t + 1):
            M = M + prod(i + 1, t) @ (beta[i] * np.outer(k[i], v[i]))
        o[t] = M.T @ q[t]
    S_T = prod(0, T - 1) @ S0
    for i in range(T):
        S_T = S_T + prod(i + 1, T - 1) @ (beta[i] * np.outer(k[i], v[i]))
    return o, S_T


def dplr_unrolled(q, k, v, a, b, alpha, S0=None):
    """Brute force for the general DPLR recurrence: explicit d_k x d_k transitions
    A_j = Diag(alpha_j) - a_j b_j^T and o_t = q_t^T [(A_t...A_1) S0 + sum_i (A_t...A_{i+1}) k_i v_i^T]
    (Rationalist Deep-Dive, section 3.2 "DPLR Structure")."""
    T, dk = q.shape
    dv = v.shape[1]
    S0 = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    eye = np.eye(dk)
    A = [np.diag(alpha[j]) - np.outer(a[j], b[j]) for j in range(T)]

    def prod(lo, hi):
        P = eye.copy()
        for j in range(lo, hi + 1):
            P = A[j] @ P
        return P

    o = np.zeros((T, dv))
    for t in range(T):
        M = prod(0, t) @ S0
        for i in range(t + 1):
            M = M + prod(i + 1, t) @ np.outer(k[i], v[i])
        o[t] = M.T @ q[t]
    S_T = prod(0, T - 1) @ S0
    for i in range(T):
        S_T = S_T + prod(i + 1, T - 1) @ np.outer(k[i], v[i])
    return o, S_T

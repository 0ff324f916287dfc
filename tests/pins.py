"""Pins for the KDA oracle: checks against what the pages and the mathematics fix.

Each ``pin_*`` function takes ``fwd`` (a callable with the signature of
``oracle.oracle_forward``) and raises AssertionError when the implementation
disagrees with its pin. The pin tests call them on the oracle; the mutation
test calls them on deliberately broken copies of the oracle to show that every
plausible mistake fails at least one pin.

Sources (Kimi Linear summaries):
  * worked two-channel decay table: docsaid.org, "KDA: Splitting the Decay
    Across Channels" (only the forget step);
  * reductions: alpha = 1 gives DeltaNet, a per-head scalar gate gives Gated
    DeltaNet ("Rationalist Deep-Dive" sections 2.2-2.3; summary section 2.2);
    beta = 0 leaves a pure per-channel decay, and the small-erase limit is GLA
    (docsaid.org, remark on GLA);
  * delta rule reaches its target: with beta = 1 and a unit key, the update is
    an exact gradient step to zero loss, so S_t^T k_t = v_t ("Rationalist
    Deep-Dive" section 2.2); this also fixes the order "decay, then correct"
    (summary section 3);
  * unrolled form with explicit transition products (section 3.3 and the
    summary's section 6.1, beta restored);
  * contraction: with unit k, alpha <= 1 and beta in [0, 1] the transition has
    spectral norm <= 1, so ||S_t||_F <= ||S_{t-1}||_F + beta_t ||v_t||.
"""

from __future__ import annotations

import json
import os

import numpy as np

from refs import textbook

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _one_head(fwd, q, k, v, beta, log_alpha, S0=None):
    T = q.shape[0]
    o, hT = fwd(q[:, None, :], k[:, None, :], v[:, None, :], log_alpha[:, None, :],
                beta[:, None], h0=None if S0 is None else S0[None, None])
    return o[:, 0, :], hT[0, 0]


def _draw(rng, T, dk, dv, unit_k=True, unit_q=True):
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    if unit_q:
        q /= np.linalg.norm(q, axis=1, keepdims=True)
    if unit_k:
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    x = rng.standard_normal((T, dk)) + 1.0
    log_alpha = -np.log1p(np.exp(-x))
    S0 = 0.3 * rng.standard_normal((dk, dv))
    # the oracle reads fp32 inputs; round once here so every reference sees the same values
    f = lambda a: np.asarray(a, dtype=np.float32).astype(np.float64)
    return f(q), f(k), f(v), f(beta), f(log_alpha), S0


def pin_decay_table(fwd):
    """Printed worked example: Diag(alpha) S on the state [8, 6]."""
    with open(os.path.join(GOLDEN, "decay_table.json")) as fh:
        g = json.load(fh)
    S0 = np.array(g["state_before"], dtype=np.float64)[:, None]     # dk=2, dv=1
    for case in g["cases"]:
        alpha = np.array(case["alpha"], dtype=np.float64)
        # one token with beta = 0: only the forget step acts on the state
        q = np.array([[1.0, 0.0]])
        k = np.array([[0.6, 0.8]])
        v = np.array([[0.0]])
        la = np.log(alpha)[None, :]
        _, S1 = _one_head(fwd, q, k, v, np.array([0.0]), la, S0)
        np.testing.assert_allclose(S1[:, 0], case["state_after"], rtol=1e-7, atol=1e-12,
                                   err_msg=case["label"])


def pin_deltanet(fwd, seed=1):
    """alpha = 1 reduces KDA to DeltaNet (written as SGD on the reconstruction loss)."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, _, S0 = _draw(rng, 12, 4, 3)
    la = np.zeros_like(q)
    o, S = _one_head(fwd, q, k, v, beta, la, S0)
    o_ref, S_ref = textbook.deltanet_gradient_step(q, k, v, beta, S0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12, atol=1e-12)


def pin_gated_deltanet(fwd, seed=2):
    """alpha constant across channels reduces KDA to scalar-gated Gated DeltaNet."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, _, S0 = _draw(rng, 12, 4, 3)
    a = np.asarray(np.exp(-rng.random(12) * 0.7), dtype=np.float64)
    la = np.repeat(np.log(a)[:, None], 4, axis=1).astype(np.float32).astype(np.float64)
    a = np.exp(la[:, 0])
    o, S = _one_head(fwd, q, k, v, beta, la, S0)
    o_ref, S_ref = textbook.gated_deltanet_scalar(q, k, v, beta, a, S0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12, atol=1e-12)


def pin_identity_step(fwd, seed=3):
    """alpha = 1 and beta = 0: the state never changes and o_t = S0^T q_t."""
    rng = np.random.default_rng(seed)
    q, k, v, _, _, S0 = _draw(rng, 9, 4, 3)
    o, S = _one_head(fwd, q, k, v, np.zeros(9), np.zeros_like(q), S0)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(o, q @ S0, rtol=1e-13, atol=1e-14)


def pin_pure_decay(fwd, seed=4):
    """beta = 0: S_t = Diag(alpha_t) S_{t-1} exactly (GLA's transition with no write)."""
    rng = np.random.default_rng(seed)
    q, k, v, _, la, S0 = _draw(rng, 7, 4, 3)
    o, S = _one_head(fwd, q, k, v, np.zeros(7), la, S0)
    S_ref = S0.copy()
    o_ref = np.zeros_like(o)
    for t in range(7):
        S_ref = np.exp(la[t])[:, None] * S_ref
        o_ref[t] = S_ref.T @ q[t]
    np.testing.assert_allclose(S, S_ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-14)


def pin_reaches_target(fwd, seed=5):
    """beta = 1 and ||k|| = 1: after each update S_t^T k_t = v_t (zero loss).

    Only 'decay first, then correct' has this property when alpha varies by
    channel, so it also pins the order of the two factors.
    """
    rng = np.random.default_rng(seed)
    T, dk, dv = 6, 4, 3
    q, k, v, _, la, S0 = _draw(rng, T, dk, dv)
    # use the state after t tokens: run prefixes and check the last token's target
    for t in range(1, T + 1):
        _, S = _one_head(fwd, q[:t], k[:t], v[:t], np.ones(t), la[:t], S0)
        kt = k[t - 1] / np.linalg.norm(k[t - 1])
        # k is fp32-rounded; rescale S^T k by ||k||^2 error bound
        np.testing.assert_allclose(S.T @ k[t - 1], v[t - 1], rtol=0,
                                   atol=1e-6 * (1 + np.abs(v[t - 1]).max()))
        del kt


def pin_gla_limit(fwd, seed=6, eps=1e-6):
    """Erase strength -> 0 with the write held fixed gives GLA: beta = eps, v = v/eps."""
    rng = np.random.default_rng(seed)
    q, k, v, _, la, S0 = _draw(rng, 10, 4, 3)
    beta = np.full(10, eps)
    o, S = _one_head(fwd, q, k, v / eps, beta, la, S0)
    o_ref, S_ref = textbook.gla(q, k, v, np.exp(la), S0)
    # the difference is the erase term, O(eps) times the state's size
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-4)
    np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-4)


def pin_unrolled(fwd, seed=7):
    """Brute force: explicit products of d_k x d_k transitions (tiny T)."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, la, S0 = _draw(rng, 6, 4, 3)
    o, S = _one_head(fwd, q, k, v, beta, la, S0)
    o_ref, S_ref = textbook.kda_unrolled(q, k, v, beta, np.exp(la), S0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-11, atol=1e-12)


def pin_square_state_unrolled(fwd, seed=8):
    """Same brute force with d_k = d_v and a non-symmetric S0 (catches transposes)."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, la, _ = _draw(rng, 5, 4, 4)
    S0 = np.arange(16, dtype=np.float64).reshape(4, 4) / 10.0
    o, S = _one_head(fwd, q, k, v, beta, la, S0)
    o_ref, S_ref = textbook.kda_unrolled(q, k, v, beta, np.exp(la), S0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-11, atol=1e-12)


def pin_contraction(fwd, seed=9, T=40):
    """||S_t||_F <= ||S_{t-1}||_F + beta_t ||v_t|| with unit k, alpha <= 1, beta in [0, 1]."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, la, S0 = _draw(rng, T, 4, 3)
    # renormalise k in fp64 so ||k|| = 1 exactly up to fp64 rounding
    k = k / np.linalg.norm(k, axis=1, keepdims=True)
    prev = np.linalg.norm(S0)
    for t in range(1, T + 1):
        _, S = _one_head(fwd, q[:t], k[:t], v[:t], beta[:t], la[:t], S0)
        cur = np.linalg.norm(S)
        assert cur <= prev + beta[t - 1] * np.linalg.norm(v[t - 1]) + 1e-6, (t, cur, prev)
        prev = cur


ALL_PINS = [pin_decay_table, pin_deltanet, pin_gated_deltanet, pin_identity_step,
            pin_pure_decay, pin_reaches_target, pin_gla_limit, pin_unrolled,
            pin_square_state_unrolled, pin_contraction]


# ---------------------------------------------------------------------------
# Pins for the Gated DeltaNet oracle (one scalar gate a_t per token and head;
# "Rationalist Deep-Dive" section 2.3, summary section 2.2). Each takes ``gfwd``
# with the signature of ``oracle.oracle_gdn_forward``.
# ---------------------------------------------------------------------------

def _gdn_one_head(gfwd, q, k, v, beta, log_a, S0=None):
    o, hT = gfwd(q[:, None, :], k[:, None, :], v[:, None, :], log_a[:, None], beta[:, None],
                 h0=None if S0 is None else S0[None, None])
    return o[:, 0, :], hT[0, 0]


def _gdn_draw(rng, T, dk, dv):
    q, k, v, beta, _, S0 = _draw(rng, T, dk, dv)
    log_a = np.asarray(-rng.random(T) * 0.7, dtype=np.float32).astype(np.float64)
    return q, k, v, beta, log_a, S0


def pin_gdn_textbook(gfwd, seed=21):
    """Against the textbook Gated DeltaNet loop, S <- a (I - beta k k^T) S + beta k v^T."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, log_a, S0 = _gdn_draw(rng, 12, 4, 3)
    o, S = _gdn_one_head(gfwd, q, k, v, beta, log_a, S0)
    o_ref, S_ref = textbook.gated_deltanet_scalar(q, k, v, beta, np.exp(log_a), S0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12, atol=1e-12)


def pin_gdn_deltanet(gfwd, seed=22):
    """a = 1 reduces Gated DeltaNet to DeltaNet (one gradient step per token)."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, _, S0 = _gdn_draw(rng, 10, 4, 3)
    o, S = _gdn_one_head(gfwd, q, k, v, beta, np.zeros(10), S0)
    o_ref, S_ref = textbook.deltanet_gradient_step(q, k, v, beta, S0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12, atol=1e-12)


def pin_gdn_pure_gate(gfwd, seed=23):
    """beta = 0: S_t = a_t S_{t-1} exactly, o_t = S_t^T q_t."""
    rng = np.random.default_rng(seed)
    q, k, v, _, log_a, S0 = _gdn_draw(rng, 7, 4, 3)
    o, S = _gdn_one_head(gfwd, q, k, v, np.zeros(7), log_a, S0)
    S_ref = S0.copy()
    for t in range(7):
        S_ref = np.exp(log_a[t]) * S_ref
        np.testing.assert_allclose(o[t], S_ref.T @ q[t], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S, S_ref, rtol=1e-13, atol=1e-15)


def pin_gdn_reaches_target(gfwd, seed=24):
    """beta = 1 and a unit key: after each token S_t^T k_t = v_t (the gated erase removes
    the old value along k completely, then the write puts v_t there)."""
    rng = np.random.default_rng(seed)
    q, k, v, _, log_a, S0 = _gdn_draw(rng, 6, 4, 3)
    for t in range(1, 7):
        _, S = _gdn_one_head(gfwd, q[:t], k[:t], v[:t], np.ones(t), log_a[:t], S0)
        np.testing.assert_allclose(S.T @ k[t - 1], v[t - 1], rtol=0,
                                   atol=1e-6 * (1 + np.abs(v[t - 1]).max()))


def pin_gdn_heads_and_sequences(gfwd, seed=25):
    """Several heads and a packed batch: each (sequence, head) equals its own textbook
    loop (catches a gate read from the wrong token or head)."""
    rng = np.random.default_rng(seed)
    H, dk, dv, lens = 3, 4, 3, [5, 0, 7]
    T = sum(lens)
    f = lambda a: np.asarray(a, dtype=np.float32).astype(np.float64)
    q = f(rng.standard_normal((T, H, dk)))
    k = rng.standard_normal((T, H, dk))
    k = f(k / np.linalg.norm(k, axis=2, keepdims=True))
    v = f(rng.standard_normal((T, H, dv)))
    beta = f(1.0 / (1.0 + np.exp(-rng.standard_normal((T, H)))))
    log_a = f(-rng.random((T, H)) * 0.9)
    h0 = 0.3 * rng.standard_normal((len(lens), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    o, hT = gfwd(q, k, v, log_a, beta, h0=h0, cu_seqlens=cu)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        for h in range(H):
            o_ref, S_ref = textbook.gated_deltanet_scalar(q[a:b, h], k[a:b, h], v[a:b, h],
                                                          beta[a:b, h], np.exp(log_a[a:b, h]),
                                                          h0[n, h])
            np.testing.assert_allclose(o[a:b, h], o_ref, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(hT[n, h], S_ref, rtol=1e-12, atol=1e-12)


ALL_GDN_PINS = [pin_gdn_textbook, pin_gdn_deltanet, pin_gdn_pure_gate, pin_gdn_reaches_target,
                pin_gdn_heads_and_sequences]


# ---------------------------------------------------------------------------
# Pins for the general DPLR oracle (Rationalist Deep-Dive, section 3.2; summary
# section 6.2). Each takes ``dfwd`` with the signature of ``oracle.oracle_dplr_forward``.
# ---------------------------------------------------------------------------

def _dplr_one_head(dfwd, q, k, v, a, b, log_alpha, S0=None):
    o, hT = dfwd(q[:, None], k[:, None], v[:, None], a[:, None], b[:, None],
                 log_alpha[:, None], h0=None if S0 is None else S0[None, None])
    return o[:, 0], hT[0, 0]


def _dplr_draw(rng, T, dk, dv):
    q, k, v, _, la, S0 = _draw(rng, T, dk, dv)
    f = lambda x: np.asarray(x, dtype=np.float32).astype(np.float64)
    a = f(0.5 * rng.standard_normal((T, dk)) / np.sqrt(dk))
    b = f(0.5 * rng.standard_normal((T, dk)) / np.sqrt(dk))
    return q, k, v, a, b, la, S0


def pin_dplr_unrolled(dfwd, seed=31):
    """Brute force: explicit products of Diag(alpha) - a b^T (catches a transposed
    low-rank term, a and b swapped, the read of the decayed state)."""
    rng = np.random.default_rng(seed)
    q, k, v, a, b, la, S0 = _dplr_draw(rng, 6, 4, 3)
    o, S = _dplr_one_head(dfwd, q, k, v, a, b, la, S0)
    o_ref, S_ref = textbook.dplr_unrolled(q, k, v, a, b, np.exp(la), S0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-11, atol=1e-12)


def pin_dplr_without_correction_is_gla(dfwd, seed=32):
    """a = 0: no low-rank correction, the per-channel decay and an additive write (GLA)."""
    rng = np.random.default_rng(seed)
    q, k, v, _, b, la, S0 = _dplr_draw(rng, 9, 4, 3)
    o, S = _dplr_one_head(dfwd, q, k, v, np.zeros_like(b), b, la, S0)
    o_ref, S_ref = textbook.gla(q, k, v, np.exp(la), S0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12, atol=1e-12)


def pin_dplr_tied_factors_are_kda(dfwd, seed=33):
    """a = beta k, b = k * alpha and the value scaled by beta give KDA (the DPLR form of
    the KDA update in Deep-Dive section 3.2, with beta on the write as in summary
    section 3): the result equals the textbook KDA brute force."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, la, S0 = _draw(rng, 7, 4, 3)
    alpha = np.exp(la)
    a = beta[:, None] * k
    b = k * alpha
    o, S = _dplr_one_head(dfwd, q, k, beta[:, None] * v, a, b, la, S0)
    o_ref, S_ref = textbook.kda_unrolled(q, k, v, beta, alpha, S0)
    # (a, b and beta v are formed in fp64 here and rounded to fp32 by the oracle's input
    #  conversion: agreement to ~1e-7 relative, against O(1) for a wrong formula)
    np.testing.assert_allclose(o, o_ref, rtol=2e-6, atol=1e-9)
    np.testing.assert_allclose(S, S_ref, rtol=2e-6, atol=1e-9)


ALL_DPLR_PINS = [pin_dplr_unrolled, pin_dplr_without_correction_is_gla,
                 pin_dplr_tied_factors_are_kda]

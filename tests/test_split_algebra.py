"""The algebra of the time split, checked on the CPU with the fp64 oracle as the primitive.

Every step of the KDA recurrence (Kimi Linear summary, section 3) is affine in the state:
S_t = A_t S_{t-1} + B_t with A_t = (I - beta_t k_t k_t^T) Diag(alpha_t) and B_t = beta_t k_t v_t^T.
So a run of tokens maps its entering state S to M S + R, where M is the product of its A_t
(the run from the identity with v = 0) and R is its final state from a zero start; and its
output is the output from a zero start plus the output of the same run from S with v = 0.
The time-split prefill evaluates exactly this: every segment from a zero state at once, the
transitions, a scan S_{j+1} = M_j S_j + R_j over the segments, and a correction pass that
adds each segment's dependence on the state entering it. Here the decomposition, composed
from oracle runs, must equal the single pass over the whole sequence to fp64 rounding.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import kda_inputs
import oracle


def _run(x, a, b, h0=None, v_zero=False, dv=None):
    """Oracle over tokens [a, b) of head-batched inputs x; v replaced by zeros if asked."""
    sl = {n: x[n][a:b] for n in ("q", "k", "v", "log_alpha", "beta")}
    if v_zero:
        T, H, _ = sl["q"].shape
        sl["v"] = torch.zeros((T, H, dv), dtype=torch.float32)
    return oracle.oracle_forward(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"], h0=h0)


@pytest.mark.parametrize("bounds", [(0, 128, 192, 320), (0, 64, 65, 200, 333)])
def test_time_split_decomposition_equals_the_single_pass(bounds):
    T, H, d = bounds[-1], 2, 128
    x = kda_inputs.make_prefill([T], H, torch.float32, torch.float32, x_mean=3.0, h0=True,
                                seed=len(bounds), h0_std=0.5)
    o_ref, hT_ref = oracle.oracle_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                          h0=x["h0"])
    n = len(bounds) - 1
    eye = torch.eye(d, dtype=torch.float64).expand(1, H, d, d).contiguous()
    o = np.zeros_like(o_ref)
    # zero-state pass: segment 0 from h0, the others from zero; the transitions M_j
    R, M = [], [None] * n
    for j in range(n):
        a, b = bounds[j], bounds[j + 1]
        o_z, r = _run(x, a, b, h0=x["h0"] if j == 0 else None)
        o[a:b] = o_z
        R.append(r)
        if 0 < j < n - 1:
            _, M[j] = _run(x, a, b, h0=eye, v_zero=True, dv=d)
    # scan: the state entering each segment
    S = [None, R[0]]
    for j in range(1, n - 1):
        S.append(np.einsum("hik,hkv->hiv", M[j][0], S[j][0])[None] + R[j])
    # correction pass: each later segment from its entering state with v = 0
    hT = R[n - 1].copy()
    for j in range(1, n):
        a, b = bounds[j], bounds[j + 1]
        o_c, s_c = _run(x, a, b, h0=torch.from_numpy(S[j]), v_zero=True, dv=d)
        o[a:b] += o_c
        if j == n - 1:
            hT += s_c
    assert np.abs(o - o_ref).max() <= 1e-12 * np.abs(o_ref).max()
    assert np.abs(hT - hT_ref).max() <= 1e-12 * np.abs(hT_ref).max()


def test_transition_is_the_product_of_the_steps():
    """M of a short run, from the identity with v = 0, equals the explicit product of
    A_t = (I - beta_t k_t k_t^T) Diag(alpha_t), applied in token order."""
    T, H, d = 6, 1, 128
    x = kda_inputs.make_prefill([T], H, torch.float32, torch.float32, x_mean=1.0, seed=3)
    eye = torch.eye(d, dtype=torch.float64).expand(1, H, d, d).contiguous()
    _, M = _run(x, 0, T, h0=eye, v_zero=True, dv=d)
    P = np.eye(d)
    for t in range(T):
        k = x["k"][t, 0].double().numpy()
        a = np.exp(x["log_alpha"][t, 0].double().numpy())
        b = float(x["beta"][t, 0])
        P = (np.eye(d) - b * np.outer(k, k)) @ np.diag(a) @ P
    assert np.abs(M[0, 0] - P).max() <= 1e-12

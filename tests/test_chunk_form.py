"""The chunkwise WY/UT algebra equals the token recurrence (fp64, CPU).

This proves the derivation the CUDA chunk kernels implement before any kernel
runs: the chunk form is an exact re-association of the recurrence, so the two
differ only by fp64 rounding.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import kda_inputs
import oracle
from refs import chunk_form


def _inputs(T, x_mean=3.0, seed=0, d=128, H=1):
    inp = kda_inputs.make_prefill([T], H, torch.float32, torch.float32, x_mean, True, seed,
                                  "cpu", d=d)
    return inp


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_chunk_form_equals_recurrence(T):
    inp = _inputs(T, seed=T)
    o_ref, s_ref = oracle.oracle_forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                         inp["beta"], h0=inp["h0"])
    f = lambda x: x[:, 0].double().numpy()
    o, s = chunk_form.chunk_forward(f(inp["q"]), f(inp["k"]), f(inp["v"]),
                                    inp["beta"][:, 0].double().numpy(), f(inp["log_alpha"]),
                                    S0=inp["h0"][0, 0].double().numpy())
    scale_o = np.abs(o_ref).max()
    scale_s = np.abs(s_ref).max()
    assert np.abs(o - o_ref[:, 0]).max() <= 1e-12 * scale_o
    assert np.abs(s - s_ref[0, 0]).max() <= 1e-12 * scale_s


def test_chunk_form_strong_decay():
    """log alpha near -5 per step: per-chunk decay reaches hundreds of nats (fp64 still exact)."""
    inp = _inputs(150, x_mean=-5.0, seed=5)
    o_ref, s_ref = oracle.oracle_forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                         inp["beta"], h0=inp["h0"])
    f = lambda x: x[:, 0].double().numpy()
    o, s = chunk_form.chunk_forward(f(inp["q"]), f(inp["k"]), f(inp["v"]),
                                    inp["beta"][:, 0].double().numpy(), f(inp["log_alpha"]),
                                    S0=inp["h0"][0, 0].double().numpy())
    assert np.abs(o - o_ref[:, 0]).max() <= 1e-12 * np.abs(o_ref).max()
    assert np.abs(s - s_ref[0, 0]).max() <= 1e-12 * max(np.abs(s_ref).max(), 1e-300)


def test_forward_substitution_inverse():
    rng = np.random.default_rng(0)
    A = np.tril(rng.standard_normal((64, 64)) * 0.2, -1)
    T = chunk_form.forward_substitution_inverse(A)
    np.testing.assert_allclose(T @ (np.eye(64) + A), np.eye(64), atol=1e-10)


def test_dplr_chunk_form_matches_the_dplr_oracle():
    """The general DPLR chunk algebra (four decayed Grams) reproduces the token-by-token
    DPLR oracle to fp64 rounding, across chunk boundaries and a ragged last chunk."""
    import oracle
    from refs.chunk_form import dplr_chunked
    rng = np.random.default_rng(41)
    T, dk, dv = 200, 16, 8
    f = lambda x: np.asarray(x, dtype=np.float32).astype(np.float64)
    q, k = f(rng.standard_normal((T, dk)) / 4), f(rng.standard_normal((T, dk)) / 4)
    v = f(rng.standard_normal((T, dv)))
    a, b = f(rng.standard_normal((T, dk)) / 4), f(rng.standard_normal((T, dk)) / 4)
    la = f(-np.log1p(np.exp(-(rng.standard_normal((T, dk)) + 2.0))))
    S0 = 0.3 * rng.standard_normal((dk, dv))
    o_ref, S_ref = oracle.oracle_dplr_forward(q[:, None], k[:, None], v[:, None], a[:, None],
                                              b[:, None], la[:, None], h0=S0[None, None])
    for C in (64, 16):
        o, S = dplr_chunked(q, k, v, a, b, la, S0, C=C)
        np.testing.assert_allclose(o, o_ref[:, 0], rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(S, S_ref[0, 0], rtol=1e-9, atol=1e-11)

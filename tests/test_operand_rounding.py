"""The tensor-core kernel's operand precision, checked on the CPU.

The kernel evaluates the chunk form in an end-of-chunk factorisation and rounds the
operands of its products to bf16 (Rk, Rq, Ck, V, T*beta, S'', W', P, Delta), with fp32
accumulators and an fp32 state. `refs.rounded_chunk` evaluates the same algebra in fp64
with a rounding hook at every operand. These tests show (1) that the factorisation is
exact (hooks off: equal to the token recurrence to fp64 rounding) and (2) that the
kernel's roundings stay inside the bf16 parity bound on inputs drawn like the 4,096-token
prefill workload, and that raising every operand to tf32 shrinks the error as its three
extra mantissa bits should.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import kda_inputs
import oracle
from refs import rounded_chunk as rc

TOL_BF16 = 2e-2


def _draw(T, h0_std=0.02, x_mean=3.0, seed=0):
    x = kda_inputs.make_prefill([T], 1, torch.bfloat16, torch.float32, x_mean, True, seed, "cpu",
                                h0_std=h0_std)
    o_ref, s_ref = oracle.oracle_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                         h0=x["h0"])
    f = lambda t: t[:, 0].double().numpy()
    args = (f(x["q"]), f(x["k"]), f(x["v"]), x["beta"][:, 0].double().numpy(),
            f(x["log_alpha"]), x["h0"][0, 0].double().numpy())
    return args, np.asarray(o_ref)[:, 0], np.asarray(s_ref)[0, 0]


def _err(x, ref):
    return float(np.abs(x - ref).max() / np.abs(ref).max())


@pytest.mark.parametrize("T", [64, 200])
def test_factorised_form_is_exact(T):
    args, o_ref, s_ref = _draw(T, h0_std=1.0, seed=T)
    o, s = rc.chunk_forward_rounded(*args)
    assert _err(o, o_ref) <= 1e-12
    assert _err(s, s_ref) <= 1e-12


def test_bf16_operands_within_bound_and_tf32_tighter():
    args, o_ref, s_ref = _draw(1024, seed=7)
    bf = dict(tiles=rc.round_bf16, t_beta=rc.round_bf16, state=rc.round_bf16,
              left=rc.round_bf16, update=rc.round_bf16, acc=rc.as_f32, out=rc.round_bf16)
    o_b, s_b = rc.chunk_forward_rounded(*args, **bf)
    e_ob, e_sb = _err(o_b, o_ref), _err(s_b, s_ref)
    assert e_ob <= TOL_BF16 and e_sb <= TOL_BF16
    tf = {n: (rc.round_tf32 if f is rc.round_bf16 and n != "out" else f) for n, f in bf.items()}
    o_t, s_t = rc.chunk_forward_rounded(*args, **tf)
    # three more mantissa bits: the state's error falls several-fold (ideally 8x)
    assert _err(s_t, s_ref) <= e_sb / 3

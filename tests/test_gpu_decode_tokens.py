"""GPU parity of the multi-token decode step (kda_decode_tokens) through the C ABI.

kda_decode_tokens applies the recurrence to t new tokens of every sequence with the
state read once and written once. It is checked against the fp64 oracle (the same
token recurrence, sequence by sequence) within the dtype's bound, and against t
consecutive single steps (kda_decode_step), whose per-token arithmetic it repeats in
the same order: the two agree bit for bit.

Error metric and bounds as in test_gpu_parity.py: max|x - x_ref| / max|x_ref|, 1e-4
for fp32 inputs, 2e-2 for bf16 inputs with an fp32 state.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import kda_inputs
import oracle

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def rel_err(x, ref):
    x = x.detach().double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)
    ref = np.asarray(ref)
    den = np.abs(ref).max()
    return float(np.abs(x - ref).max() / (den if den > 0 else 1.0))


@pytest.fixture(scope="module")
def kda():
    from channel_wise_gated_b200 import build
    build.build()
    import channel_wise_gated_b200 as m
    return m


@pytest.fixture(autouse=True)
def _no_device_error(kda):
    yield
    assert kda.device_status() == 0


def seq_major(x):
    """[t, N, ...] (step-major, as drawn) -> [N, t, ...] contiguous (the ABI layout)."""
    return x.transpose(0, 1).contiguous()


def _draw(n_seqs, n_heads, t, qkv_dtype, gate_dtype, seed):
    dec = kda_inputs.make_decode(n_seqs, n_heads, t, qkv_dtype, gate_dtype, seed=seed,
                                 device="cuda")
    lay = {n: seq_major(dec[n]) for n in ("q", "k", "v", "log_alpha", "beta")}
    return dec, lay


@pytest.mark.parametrize("t", [1, 3, 16])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_tokens_vs_oracle(kda, t, dtype):
    dec, lay = _draw(5, 3, t, dtype, dtype, seed=100 + t)
    state = dec["state"].clone()
    o = kda.decode_tokens(lay["q"], lay["k"], lay["v"], lay["log_alpha"], lay["beta"], state)
    o_ref, s_ref = oracle.oracle_decode_steps(dec["q"], dec["k"], dec["v"], dec["log_alpha"],
                                              dec["beta"], dec["state"])
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert rel_err(o.transpose(0, 1), o_ref) <= tol
    assert rel_err(state, s_ref) <= tol


@pytest.mark.parametrize("t", [2, 5])
@pytest.mark.parametrize("gates", [torch.float32, torch.bfloat16])
def test_decode_tokens_equals_single_steps(kda, t, gates):
    """Bit-identical to t calls of kda_decode_step, both gate dtypes."""
    dec, lay = _draw(7, 5, t, torch.bfloat16, gates, seed=120 + t)
    s_multi = dec["state"].clone()
    o_multi = kda.decode_tokens(lay["q"], lay["k"], lay["v"], lay["log_alpha"], lay["beta"],
                                s_multi)
    s_step = dec["state"].clone()
    o_step = torch.stack([kda.decode_step(dec["q"][s], dec["k"][s], dec["v"][s],
                                          dec["log_alpha"][s], dec["beta"][s], s_step)
                          for s in range(t)], dim=1)
    assert torch.equal(o_multi, o_step)
    assert torch.equal(s_multi, s_step)


@pytest.mark.parametrize("t,qkv,gates", [(2, torch.bfloat16, torch.bfloat16),
                                          (4, torch.bfloat16, torch.float32),
                                          (4, torch.float32, torch.float32),
                                          (9, torch.float32, torch.bfloat16),
                                          (12, torch.bfloat16, torch.bfloat16)])
def test_decode_tokens_many_chains_equal_single_steps(kda, t, qkv, gates):
    """More (sequence, head) states than resident CTAs, so every CTA runs several in turn:
    with and without the next state's input prefetch (the launcher prefetches from three
    tokens on while two CTAs still fit an SM: not at t = 2, nor at t = 9 with fp32
    inputs, nor at t = 12), still bit-identical to single steps."""
    dec, lay = _draw(40, 16, t, qkv, gates, seed=160 + t)
    s_multi = dec["state"].clone()
    o_multi = kda.decode_tokens(lay["q"], lay["k"], lay["v"], lay["log_alpha"], lay["beta"],
                                s_multi)
    s_step = dec["state"].clone()
    o_step = torch.stack([kda.decode_step(dec["q"][s], dec["k"][s], dec["v"][s],
                                          dec["log_alpha"][s], dec["beta"][s], s_step)
                          for s in range(t)], dim=1)
    assert torch.equal(o_multi, o_step)
    assert torch.equal(s_multi, s_step)


def test_decode_tokens_full_batch(kda):
    """The multi-token decode workload that bench.py times: 256 sequences x 32 heads,
    4 tokens per call, 3 calls in a row; oracle on 48 sampled chains."""
    N, H, t, calls = 256, 32, 4, 3
    dec, _ = _draw(N, H, t * calls, torch.bfloat16, torch.bfloat16, seed=140)
    state = dec["state"].clone()
    outs = []
    for c in range(calls):
        sl = {n: seq_major(dec[n][c * t:(c + 1) * t])
              for n in ("q", "k", "v", "log_alpha", "beta")}
        outs.append(kda.decode_tokens(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"],
                                      state).transpose(0, 1))
    o = torch.cat(outs)                       # [t * calls, N, H, 128]
    g = torch.Generator().manual_seed(45)
    flat = torch.randperm(N * H, generator=g)[:48]
    seqs, heads = (flat // H).tolist(), (flat % H).tolist()
    pick = lambda x: torch.stack([x[:, n, h] for n, h in zip(seqs, heads)], dim=1)[:, :, None]
    st0 = torch.stack([dec["state"][n, h] for n, h in zip(seqs, heads)])[:, None]
    o_ref, s_ref = oracle.oracle_decode_steps(pick(dec["q"]), pick(dec["k"]), pick(dec["v"]),
                                              pick(dec["log_alpha"]), pick(dec["beta"]), st0,
                                              col_block=32)
    o_gpu = pick(o)
    s_gpu = torch.stack([state[n, h] for n, h in zip(seqs, heads)])[:, None]
    assert rel_err(o_gpu, o_ref) <= TOL_BF16
    assert rel_err(s_gpu, s_ref) <= TOL_BF16


def test_decode_tokens_rejects_bad_sizes(kda):
    dec, lay = _draw(2, 2, 1, torch.bfloat16, torch.bfloat16, seed=150)
    with pytest.raises(ValueError):
        big = torch.zeros((2, 17, 2, 128), dtype=torch.bfloat16, device="cuda")
        kda.decode_tokens(big, big, big, big, torch.zeros((2, 17, 2), dtype=torch.bfloat16,
                                                          device="cuda"), dec["state"])
    lib = kda._native.load()
    p = lambda x: x.data_ptr()
    bf = kda._native.KDA_BF16
    for n_tokens in (0, 17):
        st = lib.kda_decode_tokens(p(lay["q"]), p(lay["k"]), p(lay["v"]), p(lay["log_alpha"]),
                                   p(lay["beta"]), p(dec["state"]), p(lay["q"]), 2, n_tokens, 2,
                                   bf, bf, None)
        assert st == kda._native.KDA_ERR_SHAPE

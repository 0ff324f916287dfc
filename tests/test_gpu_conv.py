"""GPU parity of the short convolution + Swish (kda_short_conv_swish) against the fp64
oracle (oracle/layer_ops.py), and of the whole producing-layer path: convolution +
Swish on q, k and v, then the fused chunk kernel (L2 norm, gates, RMSNorm, output gate),
against the oracle's composition of the same steps (Kimi Linear summary, section 4).

The convolution's only rounding is the bf16 output (at most 2^-9 relative per value),
so its bound is 5e-3 on max|y - y_ref| / max|y_ref|; the whole path uses the bf16
bound of 2e-2.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import kda_inputs
from oracle import layer_ops

pytestmark = pytest.mark.gpu

TOL_CONV = 5e-3
TOL_BF16 = 2e-2


def rel_err(x, ref):
    x = x.detach().double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)
    ref = np.asarray(ref)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


@pytest.fixture(scope="module")
def kda():
    from channel_wise_gated_b200 import build
    build.build()
    import channel_wise_gated_b200 as m
    return m


def _draw(T, C, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn((T, C), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((C, 4), generator=g, device="cuda") * 0.5).float()
    return x, w


@pytest.mark.parametrize("T,C", [(1, 8), (31, 8), (1000, 4096), (257, 384)])
def test_conv_single_sequence(kda, T, C):
    x, w = _draw(T, C, T + C)
    y = kda.short_conv_swish(x, w)
    ref = layer_ops.short_conv_swish(x.cpu(), w.cpu())
    assert rel_err(y, ref) <= TOL_CONV


def test_conv_restarts_at_sequence_boundaries(kda):
    lens = [0, 1, 2, 3, 40, 0, 31, 33, 64, 5]   # boundaries inside and across 32-token runs
    T, C = sum(lens), 256
    x, w = _draw(T, C, 9)
    cu = torch.tensor([0] + np.cumsum(lens).tolist(), dtype=torch.int32, device="cuda")
    y = kda.short_conv_swish(x, w, cu_seqlens=cu)
    ref = layer_ops.short_conv_swish(x.cpu(), w.cpu(), cu.cpu())
    assert rel_err(y, ref) <= TOL_CONV
    # the first token of every sequence sees only its own input
    a = 0
    for L in lens:
        if L:
            one = layer_ops.swish(w.cpu().double().numpy()[:, 3] * x[a].double().cpu().numpy())
            np.testing.assert_allclose(y[a].double().cpu().numpy(), one, rtol=1e-2, atol=1e-3)
        a += L


def test_conv_then_fused_chunk_against_the_layer_oracle(kda):
    lens, H = [300, 0, 129, 64], 4
    inp = kda_inputs.make_fused_prefill(lens, H, seed=12, device="cuda")
    T, C = sum(lens), H * 128
    g = torch.Generator(device="cuda").manual_seed(13)
    ws = {n: (torch.randn((C, 4), generator=g, device="cuda") * 0.5).float() for n in "qkv"}
    cu = inp["cu_seqlens"]
    conv = {n: kda.short_conv_swish(inp[src].reshape(T, C), ws[n], cu_seqlens=cu).reshape(T, H, 128)
            for n, src in (("q", "q_pre"), ("k", "k_pre"), ("v", "v"))}
    o, hT = kda.chunk_fwd_fused(conv["q"], conv["k"], conv["v"], inp["decay_pre"], inp["beta_pre"],
                                inp["gate_pre"], inp["norm_w"], h0=inp["h0"], cu_seqlens=cu)
    o_ref, h_ref, o_pre = layer_ops.fused_layer_forward(
        inp["q_pre"], inp["k_pre"], inp["v"], inp["decay_pre"], inp["beta_pre"], inp["gate_pre"],
        inp["norm_w"], h0=inp["h0"], cu_seqlens=cu.cpu(),
        conv_w={n: ws[n].cpu() for n in "qkv"}, col_block=16, return_pre_norm=True)
    rms = np.sqrt(np.mean(o_pre * o_pre, axis=-1, keepdims=True) + layer_ops.RMS_EPS)
    x = o.double().cpu().numpy()
    e_r = float(np.abs((x - o_ref) * rms).max() / np.abs(o_ref * rms).max())
    e_o, e_s = rel_err(o, o_ref), rel_err(hT, h_ref)
    print(f"conv + fused: o {e_o:.2e} (row-scaled {e_r:.2e}) hT {e_s:.2e}")
    assert e_r <= TOL_BF16 and e_s <= TOL_BF16

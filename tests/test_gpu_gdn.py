"""GPU parity of the scalar-gate (Gated DeltaNet) prefill against the fp64 oracle.

Gated DeltaNet keeps one gate per token and head (Rationalist Deep-Dive, section 2.3;
Kimi Linear summary, section 2.2): S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} +
beta_t k_t v_t^T. The kernels run it through the KDA chunk algebra with the gate
shared by every channel, so besides the oracle (written in the Gated DeltaNet order)
the results must equal the KDA entry point's on the gate broadcast to 128 channels,
bit for bit: both evaluate the same factors in the same order.

Bounds as in the KDA parity tests: max|x - x_ref| / max|x_ref| <= 1e-4 (fp32 inputs)
and <= 2e-2 (bf16 inputs, fp32 state), on o and the final state.
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


def _inputs(lens, H, dtype, x_mean=3.0, seed=0):
    return kda_inputs.make_prefill(lens, H, dtype, torch.float32, x_mean, True, seed=seed,
                                   device="cuda", scalar_gate=True)


def _gdn(kda, inp):
    cu = None if len(inp["lens"]) == 1 else inp["cu_seqlens"]
    return kda.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                             h0=inp["h0"], cu_seqlens=cu)


def _oracle(inp, heads=None):
    sel = (lambda t: t[:, heads]) if heads is not None else (lambda t: t)
    h0 = inp["h0"] if heads is None else inp["h0"][:, heads]
    return oracle.oracle_gdn_forward(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]),
                                     sel(inp["log_alpha"]), sel(inp["beta"]), h0=h0,
                                     cu_seqlens=inp["cu_seqlens"].cpu(), col_block=16)


@pytest.mark.parametrize("T", [1, 63, 64, 200, 64 * 20 + 7])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gdn_against_oracle(kda, T, dtype):
    inp = _inputs([T], 3, dtype, seed=T)
    o, hT = _gdn(kda, inp)
    o_ref, h_ref = _oracle(inp)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    e_o, e_s = rel_err(o, o_ref), rel_err(hT, h_ref)
    print(f"gdn T={T} {dtype}: o {e_o:.2e} hT {e_s:.2e}")
    assert e_o <= tol and e_s <= tol


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gdn_equals_kda_with_broadcast_gate(kda, dtype):
    inp = _inputs([64 * 9 + 30, 100, 0, 64], 4, dtype, seed=7)
    o_g, h_g = _gdn(kda, inp)
    la = inp["log_alpha"][:, :, None].expand(-1, -1, 128).contiguous()
    o_k, h_k = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], la, inp["beta"], h0=inp["h0"],
                             cu_seqlens=inp["cu_seqlens"])
    assert torch.equal(o_g, o_k)
    assert torch.equal(h_g, h_k)


def test_gdn_packed_batch_all_heads(kda):
    inp = _inputs([0, 1, 700, 64, 2000, 33], 32, torch.bfloat16, seed=11)
    o, hT = _gdn(kda, inp)
    o_ref, h_ref = _oracle(inp)
    assert rel_err(o, o_ref) <= TOL_BF16
    assert rel_err(hT, h_ref) <= TOL_BF16
    assert torch.equal(hT[0], inp["h0"][0])   # an empty sequence returns its h0


@pytest.mark.parametrize("x_mean", [3.0, -5.0])
def test_gdn_time_split(kda, x_mean):
    """One long sequence split in time (32 heads, 3 segments); with strong decay every
    chunk takes the exact path and the segment transitions vanish."""
    T, H = 64 * 60 + 9, 32
    assert len(kda.split_plan(H, T)) - 1 == 3
    inp = _inputs([T], H, torch.bfloat16, x_mean=x_mean, seed=12)
    o, hT = _gdn(kda, inp)
    heads = [0, 9, 31]
    o_ref, h_ref = _oracle(inp, heads)
    e_o, e_s = rel_err(o[:, heads], o_ref), rel_err(hT[:, heads], h_ref)
    print(f"gdn split mu={x_mean}: o {e_o:.2e} hT {e_s:.2e}")
    assert e_o <= TOL_BF16 and e_s <= max(TOL_BF16, 1e-30)
    o_1, h_1 = kda.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                 h0=inp["h0"], split=False)
    assert rel_err(o, o_1.double().cpu().numpy()) <= TOL_BF16

"""GPU parity of the general DPLR comparison kernel (kda_dplr_chunk_fwd) against the
fp64 DPLR oracle, and its reduction to KDA when the low-rank factors are tied.

General DPLR, S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T (Rationalist
Deep-Dive, section 3.2; Kimi Linear summary, section 6.2). With a = beta k, b = k * alpha
and the value scaled by beta it is the KDA recurrence, so on those inputs the DPLR
kernel must agree with the KDA CUDA-core kernel. Bounds as for KDA: 1e-4 (fp32 inputs),
2e-2 (bf16 inputs), max|x - x_ref| / max|x_ref| on o and the final state.
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
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


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


def _run(kda, inp):
    cu = None if len(inp["lens"]) == 1 else inp["cu_seqlens"]
    return kda.dplr_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"],
                              inp["log_alpha"], h0=inp["h0"], cu_seqlens=cu)


def _oracle(inp):
    return oracle.oracle_dplr_forward(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"],
                                      inp["log_alpha"], h0=inp["h0"],
                                      cu_seqlens=inp["cu_seqlens"].cpu(), col_block=16)


@pytest.mark.parametrize("lens", [[1], [64], [65], [700], [0, 130, 1, 64, 300]])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_dplr_against_oracle(kda, lens, dtype):
    inp = kda_inputs.make_dplr_prefill(lens, 3, dtype, seed=sum(lens) + 1, device="cuda")
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    e_o, e_s = rel_err(o, o_ref), rel_err(hT, h_ref)
    print(f"dplr {lens} {dtype}: o {e_o:.2e} hT {e_s:.2e}")
    assert e_o <= tol and e_s <= tol


def test_dplr_with_tied_factors_is_kda(kda):
    inp = kda_inputs.make_prefill([64 * 5 + 11], 4, torch.float32, torch.float32, 3.0, True,
                                  seed=17, device="cuda")
    beta = inp["beta"][:, :, None]
    a = (beta * inp["k"]).contiguous()
    b = (inp["k"] * torch.exp(inp["log_alpha"])).contiguous()
    o_d, h_d = kda.dplr_chunk_fwd(inp["q"], inp["k"], (beta * inp["v"]).contiguous(), a, b,
                                  inp["log_alpha"], h0=inp["h0"])
    o_k, h_k = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                             h0=inp["h0"], kernel="simt")
    assert rel_err(o_d, o_k.double().cpu().numpy()) <= TOL_F32
    assert rel_err(h_d, h_k.double().cpu().numpy()) <= TOL_F32

"""The kernels' bounded waits, made to run out on purpose (without faulting or hanging).

kda_testing_chunk_fwd_stall runs the tensor-core prefill with every wait bounded by a
short limit and with one software signal left out: prep B does not announce that chunk
c's T*beta tile is ready. The state warps' wait for it runs out, the kernel records
KDA_ERR_TIMEOUT and every role leaves. The test checks that the status is reported, that
the device error word is then clear, and that the next ordinary call on the same device
is correct (its tensor memory was freed and its barriers are fresh).
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import kda_inputs
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    from channel_wise_gated_b200 import build
    build.build()
    import channel_wise_gated_b200 as m
    return m


def _rel(x, ref):
    x = x.detach().double().cpu().numpy()
    return float(np.abs(x - ref).max() / np.abs(ref).max())


@pytest.mark.parametrize("skip_chunk", [0, 5])
def test_a_wait_that_runs_out_is_reported_and_the_device_stays_usable(kda, skip_chunk):
    lib = kda._native.load()
    T, H = 64 * 12 + 5, 4
    inp = kda_inputs.make_prefill([T], H, torch.bfloat16, torch.float32, 3.0, True, seed=77,
                                  device="cuda")
    o = torch.empty_like(inp["q"])
    hT = torch.empty((1, H, 128, 128), dtype=torch.float32, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert kda.device_status() == 0
    st = lib.kda_testing_chunk_fwd_stall(p(inp["q"]), p(inp["k"]), p(inp["v"]),
                                         p(inp["log_alpha"]), p(inp["beta"]), p(inp["h0"]), T, H,
                                         p(o), p(hT), skip_chunk, 1000, stream)
    assert st == 0
    torch.cuda.synchronize()
    assert kda.device_status() == kda._native.KDA_ERR_TIMEOUT
    assert kda.device_status() == 0   # reading clears it
    # nothing left out: the same entry is an ordinary call
    st = lib.kda_testing_chunk_fwd_stall(p(inp["q"]), p(inp["k"]), p(inp["v"]),
                                         p(inp["log_alpha"]), p(inp["beta"]), p(inp["h0"]), T, H,
                                         p(o), p(hT), -1, 1000000, stream)
    assert st == 0
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    o2, h2 = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                           h0=inp["h0"])
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    o_ref, h_ref = oracle.oracle_forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                         inp["beta"], h0=inp["h0"], col_block=16)
    for x, ref in ((o, o_ref), (o2, o_ref), (hT, h_ref), (h2, h_ref)):
        assert _rel(x, ref) <= 2e-2

"""The allocation-free prefill entry point, kda_chunk_fwd_static.

Some callers of this library cannot allocate device memory when they call it: an op
that runs as a plugin inside an inference engine which has already reserved the
GPU's memory for its own pool and hands the op only its inputs and outputs, or code
on a latency-critical path where cudaMalloc and cudaFree are ruled out because they
can synchronise the device. For them kda_chunk_fwd_static takes its scratch from a
fixed array compiled into the library.

These tests call that entry point straight through the C ABI (ctypes, raw device
pointers), twice in a row on different problems, so that the second call starts from
the scratch contents the first one left behind. Each result is checked against the
existing workspace entry point kda_chunk_fwd_ws (given a workspace allocated here
beforehand) and against the fp64 oracle, within the bf16 tolerance of the parity
tests, and no allocation may happen during the calls. The file is named so that
pytest collects it last.
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import kda_inputs
import oracle

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


def _rel(x, ref):
    x = x.detach().double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)
    ref = ref.detach().double().cpu().numpy() if isinstance(ref, torch.Tensor) else np.asarray(ref)
    return float(np.abs(x - ref).max() / np.abs(ref).max())


@pytest.fixture(scope="module")
def lib():
    from channel_wise_gated_b200 import build
    build.build()
    from channel_wise_gated_b200 import _native
    return _native.load()


def _args(inp, o, hT):
    cu = None if len(inp["lens"]) == 1 else inp["cu_seqlens"]
    T, H, _ = inp["q"].shape
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return (p(inp["q"]), p(inp["k"]), p(inp["v"]), p(inp["log_alpha"]), p(inp["beta"]),
            p(inp["h0"]), p(cu), len(inp["lens"]), T, H, 1, p(o), p(hT)), cu is not None


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _device_status(lib):
    return lib.kda_device_status(_stream())


def _outputs(inp):
    T, H, _ = inp["q"].shape
    o = torch.empty_like(inp["q"])
    hT = torch.empty((len(inp["lens"]), H, 128, 128), dtype=torch.float32, device="cuda")
    return o, hT


def _with_workspace(lib, inp):
    """The existing entry point, kda_chunk_fwd_ws, with a workspace allocated here."""
    o, hT = _outputs(inp)
    args, has_cu = _args(inp, o, hT)
    T, H, _ = inp["q"].shape
    ws_bytes = lib.kda_chunk_fwd_workspace_size(len(inp["lens"]), T, H, 1, int(has_cu))
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    assert lib.kda_chunk_fwd_ws(*args, ctypes.c_void_p(ws.data_ptr()), ws_bytes, _stream()) == 0
    torch.cuda.synchronize()
    assert _device_status(lib) == 0
    return o, hT, ws_bytes


def _oracle(inp):
    return oracle.oracle_forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                 h0=inp["h0"], cu_seqlens=inp["cu_seqlens"].cpu(), col_block=16)


def test_static_scratch_two_calls_in_a_row(lib):
    # call 1: 32 heads, one sequence split in 3 segments (8 MiB of scratch);
    # call 2: 16 heads, split in 5 segments (8 MiB), over what call 1 left behind
    problems = [
        kda_inputs.make_prefill([64 * 56 + 21], 32, torch.bfloat16, torch.float32, 3.0, True,
                                seed=91, device="cuda"),
        kda_inputs.make_prefill([64 * 100 + 33], 16, torch.bfloat16, torch.float32, 3.0, True,
                                seed=92, device="cuda"),
    ]
    expected = [_with_workspace(lib, inp) for inp in problems]
    for _, _, ws_bytes in expected:
        assert 0 < ws_bytes <= (16 << 20)   # the time split applies and fits the array
    outs = [_outputs(inp) for inp in problems]
    torch.cuda.synchronize()
    before = torch.cuda.memory_stats()["allocation.all.allocated"]
    for inp, (o, hT) in zip(problems, outs):
        args, _ = _args(inp, o, hT)
        assert lib.kda_chunk_fwd_static(*args, _stream()) == 0
    torch.cuda.synchronize()
    assert torch.cuda.memory_stats()["allocation.all.allocated"] == before
    assert _device_status(lib) == 0
    for inp, (o, hT), (o_ws, h_ws, _) in zip(problems, outs, expected):
        assert _rel(o, o_ws) <= TOL_BF16
        assert _rel(hT, h_ws) <= TOL_BF16
        o_ref, h_ref = _oracle(inp)
        assert _rel(o, o_ref) <= TOL_BF16
        assert _rel(hT, h_ref) <= TOL_BF16


def test_static_scratch_packed_batch(lib):
    # 24 sequences x 32 heads is more CTAs than SMs: the launch order goes to scratch
    inp = kda_inputs.make_prefill([64 + 9 * i for i in range(24)], 32, torch.bfloat16,
                                  torch.float32, 3.0, True, seed=93, device="cuda")
    o_ws, h_ws, ws_bytes = _with_workspace(lib, inp)
    assert ws_bytes > 0
    for _ in range(2):
        o, hT = _outputs(inp)
        args, _ = _args(inp, o, hT)
        assert lib.kda_chunk_fwd_static(*args, _stream()) == 0
        torch.cuda.synchronize()
        assert _device_status(lib) == 0
        assert _rel(o, o_ws) <= TOL_BF16
        assert _rel(hT, h_ws) <= TOL_BF16


def test_static_scratch_uneven_segments(lib):
    # 4 heads over 321 chunks, the last one ragged: 17 segments of 19 and 18 chunks
    # (the chunk count is not a multiple of the segment count), 32 slots of scratch
    # (the workspace query also covers the fused variant's split, which takes more)
    inp = kda_inputs.make_prefill([320 * 64 + 13], 4, torch.bfloat16, torch.float32, 3.0, True,
                                  seed=94, device="cuda")
    assert lib.kda_chunk_fwd_split_plan(4, 320 * 64 + 13, 0, 16 << 20, None) == 17
    o_ws, h_ws, ws_bytes = _with_workspace(lib, inp)
    assert 32 * 4 * 128 * 128 * 4 <= ws_bytes <= (16 << 20)
    o, hT = _outputs(inp)
    args, _ = _args(inp, o, hT)
    assert lib.kda_chunk_fwd_static(*args, _stream()) == 0
    torch.cuda.synchronize()
    assert _device_status(lib) == 0
    assert _rel(o, o_ws) <= TOL_BF16
    assert _rel(hT, h_ws) <= TOL_BF16
    o_ref, h_ref = _oracle(inp)
    assert _rel(o, o_ref) <= TOL_BF16
    assert _rel(hT, h_ref) <= TOL_BF16

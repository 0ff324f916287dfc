"""The roofline numerators of bench.py, recounted from the tensors the calls read and write.

bench.py divides fixed algorithmic byte counts by event-timed durations. Here those counts
must equal the bytes of the tensors the workloads actually pass to the kernels (drawn by the
same generators at a small size, with the workloads' dtypes): every input read once, every
output written once, the fp32 state read and written once per call.
"""

from __future__ import annotations

import importlib.util
import os

import torch

import kda_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _nbytes(*ts):
    return sum(t.numel() * t.element_size() for t in ts)


def test_prefill_bytes_per_token_head():
    b = _bench()
    cfg = kda_inputs.PREFILL_CONFIGS[3]          # the long-context workload's dtypes
    T, H = 96, 3
    x = kda_inputs.make_prefill([T], H, cfg.qkv_dtype, torch.float32, cfg.x_mean, False, 0)
    o = torch.empty_like(x["q"])                 # the output has q's layout and dtype
    per_token_head = _nbytes(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], o) / (T * H)
    assert per_token_head == b.PREFILL_BYTES_PER_TOKEN_HEAD == 1540


def test_decode_bytes_per_state():
    b = _bench()
    N, H, t = 5, 3, b.DECODE_TOKENS
    c = kda_inputs.DECODE_CONFIG
    x = kda_inputs.make_decode(N, H, t, c.qkv_dtype, c.gate_dtype)
    o = torch.empty_like(x["q"])
    tokens = _nbytes(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], o) / (N * H)
    state_rw = 2 * _nbytes(x["state"]) / (N * H)
    assert state_rw == 2 * b.STATE_BYTES
    assert tokens + state_rw == b.decode_tokens_bytes_per_chain(t)
    x1 = kda_inputs.make_decode(N, H, 1, c.qkv_dtype, c.gate_dtype)
    one = _nbytes(x1["q"], x1["k"], x1["v"], x1["log_alpha"], x1["beta"], torch.empty_like(x1["q"]))
    assert one / (N * H) + state_rw == b.DECODE_BYTES_PER_CHAIN == b.decode_tokens_bytes_per_chain(1)

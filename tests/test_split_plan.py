"""Host-side arithmetic of the time split (kda_chunk_fwd_split_plan), on the CPU.

The plan decides how one long bf16 sequence is cut into segments, and the kernels
read exactly the token ranges it implies. These checks run without a GPU: the
planning call with an explicit SM count touches no device.

For every head count from 1 to 148 on a 148-SM part, and chunk counts around every
multiple of the segment counts, a plan must
  * cover the sequence exactly: bounds start at 0, end at t_total, strictly increase,
    and every inner bound is a whole chunk;
  * give every segment at least 16 chunks, with lengths differing by at most one chunk
    (the last segment alone may end in a partial chunk);
  * fit the scratch it is given: (2n - 2) * H * 64 KiB.
The segment counts of a few cases are pinned to the ones measured fastest on a B200.
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest

from channel_wise_gated_b200 import _native

SMS = 148
SLOT = 128 * 128 * 4


@pytest.fixture(scope="module")
def lib():
    from channel_wise_gated_b200 import build
    build.build()
    return _native.load()


def _plan(lib, H, T, sms=SMS, ws=_native.SIZE_MAX):
    b = (ctypes.c_int64 * (_native.KDA_MAX_SEGMENTS + 1))()
    n = lib.kda_chunk_fwd_split_plan(H, T, sms, ws, b)
    return n, [int(b[i]) for i in range(n + 1)] if n >= 2 else []


def _check(H, T, n, bounds, sms, ws):
    if n == 0:
        return
    assert 2 <= n <= _native.KDA_MAX_SEGMENTS
    assert (2 * n - 2) * H * SLOT <= ws
    assert bounds[0] == 0 and bounds[-1] == T
    b = np.array(bounds)
    assert np.all(np.diff(b) > 0)
    assert np.all(b[:-1] % 64 == 0)
    chunks = np.diff(np.append(b[:-1] // 64, (T + 63) // 64))
    assert chunks.min() >= 16
    assert chunks.max() - chunks.min() <= 1


@pytest.mark.parametrize("H", list(range(1, SMS + 1)))
def test_plan_covers_sequence(lib, H):
    seen = set()
    for n_chunks in list(range(16, 400, 7)) + [512, 1000, 1024, 3000, 16384]:
        for tail in (0, 1, 63):
            T = n_chunks * 64 - (64 - tail if tail else 0)
            n, bounds = _plan(lib, H, T)
            assert n >= 0
            _check(H, T, n, bounds, SMS, _native.SIZE_MAX)
            seen.add(n)
    if H <= SMS // 3:
        assert max(seen) >= 3   # some length splits


def test_reported_case_4_heads_321_chunks(lib):
    # 4 heads and 321 chunks: 17 segments of 19 and 18 chunks (no segment past the end)
    n, bounds = _plan(lib, 4, 321 * 64)
    assert n == 17
    _check(4, 321 * 64, n, bounds, SMS, _native.SIZE_MAX)
    assert sorted(set(np.diff(bounds).tolist())) == [18 * 64, 19 * 64]


def test_headline_plan(lib):
    # 32 heads, 1,048,576 tokens: 9 segments of 1821 and 1820 chunks (two waves of 148
    # and 140 CTAs: 18.1 ms on a B200, against 19.6 for 4 segments, 20.0 for 8, 23.5
    # for 10); within the 16 MiB static array, 4 segments of 4096 chunks
    n, bounds = _plan(lib, 32, 1 << 20)
    assert n == 9
    assert np.diff(bounds).tolist() == [1821 * 64] * 4 + [1820 * 64] * 5
    n, bounds = _plan(lib, 32, 1 << 20, ws=16 << 20)
    assert n == 4
    assert np.diff(bounds).tolist() == [4096 * 64] * 4


def test_short_segments_plan_for_full_corrections(lib):
    # 32 heads, 64 chunks: segments too short for the corrections to be counted on
    # stopping early, so the plan weighs a full correction pass: 3 segments (measured:
    # 0.277 ms, against 0.288 single, 0.298 for 2 and 0.342 for 4); 1024 chunks: 4
    assert _plan(lib, 32, 4096)[0] == 3
    assert _plan(lib, 32, 65536)[0] == 4
    # 16 heads over 1M tokens: 9 segments (144 CTAs)
    assert _plan(lib, 16, 1 << 20)[0] == 9


def test_plan_fits_given_scratch(lib):
    for H in (1, 2, 3, 4, 8, 16, 32):
        for ws in (0, 3 * H * SLOT, 16 << 20, _native.SIZE_MAX):
            n, bounds = _plan(lib, H, 1 << 20, ws=ws)
            _check(H, 1 << 20, n, bounds, SMS, ws)
        assert _plan(lib, H, 1 << 20, ws=2 * H * SLOT - 1)[0] == 0   # below one split


def test_short_and_fp32_cases_do_not_split(lib):
    assert _plan(lib, 32, 64 * 31)[0] == 0      # fewer than 2 x 16 chunks
    assert _plan(lib, 32, 63)[0] == 0           # shorter than one chunk: CUDA-core kernel
    assert _plan(lib, 148, 64 * 64)[0] == 0     # every SM busy already, short segments
    assert _plan(lib, 100, 1 << 20)[0] >= 2     # 100 heads leave 48 SMs idle: waves pay
    assert _plan(lib, 32, 64 * 40)[0] == 0      # no split pays at 40 chunks
    assert lib.kda_chunk_fwd_split_plan(0, 100, SMS, 0, None) == _native.KDA_ERR_SHAPE

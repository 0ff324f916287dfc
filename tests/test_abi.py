"""The C-ABI library loads, exports every declared entry point, and validates
arguments on the host (no GPU needed: every case here returns before any CUDA
call)."""

from __future__ import annotations

import ctypes
import os
import re

import pytest

from channel_wise_gated_b200 import _native, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(kda_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _native.load()


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in ("kda_chunk_fwd", "kda_chunk_fwd_simt", "kda_decode_step", "kda_decode_tokens",
              "kda_device_status", "kda_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in kda.h but not exported"
        assert name in _native.SIGNATURES, f"{name} has no binding signature"


def test_every_exported_entry_point_is_declared(lib):
    """The reverse of the check above: nothing leaves the library under a kda_ name that
    include/kda.h does not declare (names from the dynamic symbol table of our own build)."""
    import shutil
    import subprocess
    nm = shutil.which("nm")
    if nm is None:
        pytest.skip("nm not available")
    out = subprocess.run([nm, "-D", "--defined-only", _native.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines()
                       if ln.split() and ln.split()[-1].startswith("kda_")})
    assert exported, "no kda_ symbols exported"
    assert set(exported) <= set(declared_functions()), set(exported) - set(declared_functions())


def test_profile_summaries_are_machine_readable():
    """bench.py reads the long-context call's DRAM bytes and the tensor-pipe activity,
    each with the kernel-source hash it was taken with, from the committed ncu
    summaries; all must parse and be plausible."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench_mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench_mod)
    for f in bench_mod.CHUNK_KERNEL_SOURCES:
        assert os.path.exists(os.path.join(ROOT, "channel_wise_gated_b200", "csrc", f)), f
    dram = open(os.path.join(ROOT, "profiles", "kda_chunk_tc_longctx_dram.md")).read()
    assert re.search(r"^source_hash: ([0-9a-f]{16})$", dram, re.M)
    mb = re.search(r"^longctx_call_dram_bytes: ([0-9.]+)$", dram, re.M)
    # at least the algorithmic 51.68 GB of the call, at most a few times it
    assert mb and 51.68e9 <= float(mb.group(1)) <= 4 * 51.68e9
    full = open(os.path.join(ROOT, "profiles", "kda_chunk_tc_prefill4k_full.md")).read()
    assert re.search(r"^source_hash: ([0-9a-f]{16})$", full, re.M)
    mt = re.search(r"^tensor_pipe_active_pct: ([0-9.]+)$", full, re.M)
    assert mt and 0.0 < float(mt.group(1)) <= 100.0
    assert re.fullmatch(r"[0-9a-f]{16}", bench_mod._source_hash())


def test_status_strings(lib):
    for st in range(0, -9, -1):
        s = _native.status_string(st)
        assert s.startswith("KDA_")
    assert "scratch" in _native.status_string(_native.KDA_ERR_SCRATCH)
    assert "unknown" in _native.status_string(-99)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every case fails validation first


def _chunk(lib, **over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, h0=None, cu=None, n=1, T=64, H=2,
                dt=_native.KDA_BF16, o=FAKE, hT=None, stream=None)
    args.update(over)
    return lib.kda_chunk_fwd(args["q"], args["k"], args["v"], args["la"], args["b"], args["h0"],
                             args["cu"], args["n"], args["T"], args["H"], args["dt"], args["o"],
                             args["hT"], args["stream"])


def test_chunk_validation(lib):
    assert _chunk(lib, q=None) == _native.KDA_ERR_NULL
    assert _chunk(lib, o=None) == _native.KDA_ERR_NULL
    assert _chunk(lib, H=0) == _native.KDA_ERR_SHAPE
    assert _chunk(lib, T=-1) == _native.KDA_ERR_SHAPE
    assert _chunk(lib, n=0) == _native.KDA_ERR_SHAPE
    assert _chunk(lib, dt=7) == _native.KDA_ERR_DTYPE
    assert _chunk(lib, k=FAKE + 8) == _native.KDA_ERR_ALIGN
    assert _chunk(lib, hT=FAKE + 4) == _native.KDA_ERR_ALIGN
    assert _chunk(lib, n=2, cu=None) == _native.KDA_ERR_SEQLENS
    assert lib.kda_chunk_fwd_simt(None, FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 2,
                                  _native.KDA_F32, FAKE, None, None) == _native.KDA_ERR_NULL
    # the workspace entry point: same validation, plus an aligned workspace
    ws = lib.kda_chunk_fwd_ws
    assert ws(None, FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 2, _native.KDA_BF16, FAKE, None,
              FAKE, 1 << 20, None) == _native.KDA_ERR_NULL
    assert ws(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 2, _native.KDA_BF16, FAKE, None,
              FAKE + 8, 1 << 20, None) == _native.KDA_ERR_ALIGN
    # the allocation-free entry point validates its arguments before it touches the device
    st = lib.kda_chunk_fwd_static
    assert st(None, FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 2, _native.KDA_BF16, FAKE, None,
              None) == _native.KDA_ERR_NULL
    assert st(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 0, _native.KDA_BF16, FAKE, None,
              None) == _native.KDA_ERR_SHAPE
    assert st(FAKE, FAKE + 8, FAKE, FAKE, FAKE, None, None, 1, 64, 2, _native.KDA_BF16, FAKE,
              None, None) == _native.KDA_ERR_ALIGN


def test_layer_entry_points_validation(lib):
    """The Gated DeltaNet, fused, general-DPLR and short-convolution entry points reject bad
    arguments on the host, before any CUDA call."""
    bf, f32 = _native.KDA_BF16, _native.KDA_F32
    gdn, gdn_ws = lib.kda_gdn_chunk_fwd, lib.kda_gdn_chunk_fwd_ws
    assert gdn(None, FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 2, bf, FAKE, None,
               None) == _native.KDA_ERR_NULL
    assert gdn(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 2, 5, FAKE, None,
               None) == _native.KDA_ERR_DTYPE
    assert gdn(FAKE, FAKE, FAKE, FAKE + 4, FAKE, None, None, 1, 64, 2, bf, FAKE, None,
               None) == _native.KDA_ERR_ALIGN
    assert gdn_ws(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 2, bf, FAKE, None, FAKE + 8,
                  1 << 20, None) == _native.KDA_ERR_ALIGN
    assert gdn_ws(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 3, 64, 2, bf, FAKE, None, None, 0,
                  None) == _native.KDA_ERR_SEQLENS
    # fused: q_pre, k_pre, v, decay_pre, beta_pre, gate_pre, norm_w, h0, cu, n, T, H, o, hT, ws
    fused = lambda **a: lib.kda_chunk_fwd_fused(
        a.get("q", FAKE), FAKE, FAKE, FAKE, FAKE, a.get("gate", FAKE), a.get("norm", FAKE), None,
        None, 1, 64, a.get("H", 2), FAKE, None, a.get("ws", None), 0, None)
    assert fused(q=None) == _native.KDA_ERR_NULL
    assert fused(gate=None) == _native.KDA_ERR_NULL
    assert fused(norm=None) == _native.KDA_ERR_NULL
    assert fused(gate=FAKE + 2) == _native.KDA_ERR_ALIGN
    assert fused(ws=FAKE + 8) == _native.KDA_ERR_ALIGN
    assert fused(H=0) == _native.KDA_ERR_SHAPE
    # general DPLR: q, k, v, a, b, log_alpha, h0, cu, n, T, H, dtype, o, hT
    dplr = lambda **x: lib.kda_dplr_chunk_fwd(
        FAKE, FAKE, FAKE, x.get("a", FAKE), x.get("b", FAKE), FAKE, None, None, 1, 64, 2,
        x.get("dt", f32), FAKE, None, None)
    assert dplr(a=None) == _native.KDA_ERR_NULL
    assert dplr(b=FAKE + 4) == _native.KDA_ERR_ALIGN
    assert dplr(dt=9) == _native.KDA_ERR_DTYPE
    # short convolution: x, w, cu, n_seqs, T, channels, y
    conv = lambda **x: lib.kda_short_conv_swish(
        x.get("x", FAKE), x.get("w", FAKE), x.get("cu", None), x.get("n", 1), x.get("T", 64),
        x.get("C", 256), x.get("y", FAKE + 4096), None)
    assert conv(C=12) == _native.KDA_ERR_SHAPE        # not a multiple of 8 channels
    assert conv(C=0) == _native.KDA_ERR_SHAPE
    assert conv(T=-1) == _native.KDA_ERR_SHAPE
    assert conv(n=2) == _native.KDA_ERR_SEQLENS       # several sequences need cu_seqlens
    assert conv(x=None) == _native.KDA_ERR_NULL
    assert conv(w=FAKE + 4) == _native.KDA_ERR_ALIGN
    assert conv(y=FAKE) == _native.KDA_ERR_SHAPE      # no in-place convolution
    assert conv(T=0, x=None, w=None, y=None) == _native.KDA_OK   # nothing to do


def test_workspace_size_queries(lib):
    size = lib.kda_chunk_fwd_workspace_size
    bf, f32 = _native.KDA_BF16, _native.KDA_F32
    # no time split for fp32, packed batches, short sequences or bad sizes
    assert size(1, 1 << 20, 32, f32, 0) == 0
    assert size(1, 1 << 20, 32, bf, 1) == 0
    assert size(1, 64 * 16, 32, bf, 0) == 0
    assert size(0, 1 << 20, 32, bf, 0) == 0
    assert size(1, 1 << 20, 0, bf, 0) == 0


def test_decode_validation(lib):
    f = lib.kda_decode_step
    bf = _native.KDA_BF16
    assert f(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, bf, bf, None) == _native.KDA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 2, bf, bf, None) == _native.KDA_ERR_NULL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, bf, bf, None) == _native.KDA_ERR_SHAPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 3, bf, None) == _native.KDA_ERR_DTYPE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 2, FAKE, 4, 2, bf, bf, None) == _native.KDA_ERR_ALIGN


def test_decode_tokens_validation(lib):
    f = lib.kda_decode_tokens
    bf = _native.KDA_BF16
    ok = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert f(None, *ok[1:], 4, 2, 2, bf, bf, None) == _native.KDA_ERR_NULL
    assert f(*ok[:5], None, FAKE, 4, 2, 2, bf, bf, None) == _native.KDA_ERR_NULL
    assert f(*ok, 0, 2, 2, bf, bf, None) == _native.KDA_ERR_SHAPE
    assert f(*ok, 4, 0, 2, bf, bf, None) == _native.KDA_ERR_SHAPE
    assert f(*ok, 4, _native.KDA_DECODE_MAX_TOKENS + 1, 2, bf, bf, None) == _native.KDA_ERR_SHAPE
    assert f(*ok, 4, 2, 0, bf, bf, None) == _native.KDA_ERR_SHAPE
    assert f(*ok, 4, 2, 2, 5, bf, None) == _native.KDA_ERR_DTYPE
    assert f(*ok, 4, 2, 2, bf, 9, None) == _native.KDA_ERR_DTYPE
    assert f(*ok[:5], FAKE + 4, FAKE, 4, 2, 2, bf, bf, None) == _native.KDA_ERR_ALIGN


def test_decode_token_limit_matches_header():
    text = open(HEADER).read()
    m = re.search(r"#define KDA_DECODE_MAX_TOKENS (\d+)", text)
    assert m and int(m.group(1)) == _native.KDA_DECODE_MAX_TOKENS


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_native, "_lib", None)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _native.load(str(tmp_path / "missing.so"))

"""ctypes loader and numpy wrappers for the fp64 C oracle in ``kda_oracle.c``.

Test infrastructure only (see the package docstring). The C file is compiled
with gcc + OpenMP into ``oracle/_build/libkda_oracle.so`` on first use (or by
``build_oracle()``); it is rebuilt when the source is newer than the library.

Precision: the oracle widens every stored input (fp32, or bf16 already widened
to fp32 by ``torch.Tensor.float()``, which is exact) to fp64 and computes in fp64
with libm ``exp``. Outputs are fp64 numpy arrays.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile the C oracle (gcc -O2 -fopenmp, portable x86-64 code)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str):
    """Open a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    f = lib.kda_oracle_forward
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int64] * 6 + [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    g = lib.gdn_oracle_forward
    g.restype = ctypes.c_int
    g.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int64] * 6 + [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    dp = lib.dplr_oracle_forward
    dp.restype = ctypes.c_int
    dp.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int64] * 6 + [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.kda_oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build_oracle())
    return _lib


def oracle_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def _f32(x) -> np.ndarray:
    """Exact widening of a torch tensor / array to a contiguous fp32 numpy array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu").float().contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu").double().contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def oracle_forward(q, k, v, log_alpha, beta, h0=None, cu_seqlens=None, n_threads: int = 0,
                   col_block: int = 0, lib=None):
    """Run the token recurrence for every (sequence, head).

    q, k, log_alpha: [T, H, dk]; v: [T, H, dv]; beta: [T, H];
    h0: [N, H, dk, dv] or None (zero state); cu_seqlens: [N+1] or None (one sequence).
    Returns (o [T, H, dv] fp64, hT [N, H, dk, dv] fp64).
    """
    q, k, v, la, b = (_f32(x) for x in (q, k, v, log_alpha, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    assert k.shape == (T, H, dk) and la.shape == (T, H, dk)
    assert v.shape == (T, H, dv) and b.shape == (T, H)
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    h0_arr = None if h0 is None else _f64(h0)
    if h0_arr is not None:
        assert h0_arr.shape == (N, H, dk, dv)
    o = np.zeros((T, H, dv), dtype=np.float64)
    hT = np.zeros((N, H, dk, dv), dtype=np.float64)
    lib = _load() if lib is None else lib
    rc = lib.kda_oracle_forward(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, la.ctypes.data, b.ctypes.data,
        None if h0_arr is None else h0_arr.ctypes.data, cu.ctypes.data,
        N, H, dk, dv, T, int(col_block), o.ctypes.data, hT.ctypes.data, int(n_threads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_forward failed with status {rc}")
    return o, hT


def oracle_decode_steps(q, k, v, log_alpha, beta, state, n_threads: int = 0, col_block: int = 0):
    """Run ``steps`` consecutive single-token updates for N independent sequences.

    Inputs are step-major: q, k, log_alpha [steps, N, H, dk]; v [steps, N, H, dv];
    beta [steps, N, H]; state [N, H, dk, dv] (the state before the first step).
    Returns (o [steps, N, H, dv], final state [N, H, dk, dv]) in fp64.

    This is the same recurrence as ``oracle_forward`` with each sequence's tokens
    laid out one after another; it only rearranges the inputs.
    """
    q, k, v, la, b = (_f32(x) for x in (q, k, v, log_alpha, beta))
    steps, N, H, dk = q.shape
    dv = v.shape[3]

    def seq_major(x):
        # [steps, N, ...] -> [N*steps, ...] with sequence n's tokens contiguous
        return np.ascontiguousarray(np.swapaxes(x, 0, 1).reshape((N * steps,) + x.shape[2:]))

    cu = np.arange(N + 1, dtype=np.int64) * steps
    o, hT = oracle_forward(seq_major(q), seq_major(k), seq_major(v), seq_major(la), seq_major(b),
                           h0=state, cu_seqlens=cu, n_threads=n_threads, col_block=col_block)
    o = np.swapaxes(o.reshape(N, steps, H, dv), 0, 1)
    return np.ascontiguousarray(o), hT


def oracle_gdn_forward(q, k, v, log_a, beta, h0=None, cu_seqlens=None, n_threads: int = 0,
                       col_block: int = 0, lib=None):
    """Gated DeltaNet (one scalar gate per token and head) for every (sequence, head).

    q, k: [T, H, dk]; v: [T, H, dv]; log_a, beta: [T, H]; h0: [N, H, dk, dv] or None;
    cu_seqlens: [N+1] or None. Returns (o [T, H, dv] fp64, hT [N, H, dk, dv] fp64).
    """
    q, k, v, la, b = (_f32(x) for x in (q, k, v, log_a, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    assert k.shape == (T, H, dk) and la.shape == (T, H)
    assert v.shape == (T, H, dv) and b.shape == (T, H)
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    h0_arr = None if h0 is None else _f64(h0)
    if h0_arr is not None:
        assert h0_arr.shape == (N, H, dk, dv)
    o = np.zeros((T, H, dv), dtype=np.float64)
    hT = np.zeros((N, H, dk, dv), dtype=np.float64)
    lib = _load() if lib is None else lib
    rc = lib.gdn_oracle_forward(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, la.ctypes.data, b.ctypes.data,
        None if h0_arr is None else h0_arr.ctypes.data, cu.ctypes.data,
        N, H, dk, dv, T, int(col_block), o.ctypes.data, hT.ctypes.data, int(n_threads))
    if rc != 0:
        raise RuntimeError(f"gdn_oracle_forward failed with status {rc}")
    return o, hT


def oracle_dplr_forward(q, k, v, a, b, log_alpha, h0=None, cu_seqlens=None, n_threads: int = 0,
                        col_block: int = 0, lib=None):
    """General DPLR recurrence S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T for every
    (sequence, head). q, k, a, b, log_alpha: [T, H, dk]; v: [T, H, dv]; h0, cu_seqlens as
    oracle_forward. Returns (o [T, H, dv] fp64, hT [N, H, dk, dv] fp64)."""
    q, k, v, a, b, la = (_f32(x) for x in (q, k, v, a, b, log_alpha))
    T, H, dk = q.shape
    dv = v.shape[2]
    for x in (k, a, b, la):
        assert x.shape == (T, H, dk)
    assert v.shape == (T, H, dv)
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    h0_arr = None if h0 is None else _f64(h0)
    o = np.zeros((T, H, dv), dtype=np.float64)
    hT = np.zeros((N, H, dk, dv), dtype=np.float64)
    lib = _load() if lib is None else lib
    rc = lib.dplr_oracle_forward(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, a.ctypes.data, b.ctypes.data, la.ctypes.data,
        None if h0_arr is None else h0_arr.ctypes.data, cu.ctypes.data,
        N, H, dk, dv, T, int(col_block), o.ctypes.data, hT.ctypes.data, int(n_threads))
    if rc != 0:
        raise RuntimeError(f"dplr_oracle_forward failed with status {rc}")
    return o, hT

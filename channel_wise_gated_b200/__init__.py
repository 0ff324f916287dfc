"""Kimi Delta Attention (KDA) on B200: chunkwise prefill and recurrent decode.

Thin Python binding over the C ABI of ``include/kda.h``. PyTorch is used only to
hold device memory and to name the current CUDA stream; every step of the
operator runs in the library's CUDA kernels. Functions take torch tensors,
check their dtypes, shapes and contiguity, and pass raw pointers through.

    o, hT = chunk_fwd(q, k, v, log_alpha, beta, h0=None, cu_seqlens=None)
    o     = decode_step(q, k, v, log_alpha, beta, state)      # state updated in place
    o     = decode_tokens(q, k, v, log_alpha, beta, state)    # t tokens per sequence
"""

from __future__ import annotations

from typing import Optional

import torch

from . import _native
from ._native import KdaError  # noqa: F401

D = 128

# Arithmetic type of the prefill contractions for bf16 inputs (bf16 operands, fp32 accumulation).
PREFILL_COMPUTE_DTYPE = "bf16"

_DT = {torch.float32: _native.KDA_F32, torch.bfloat16: _native.KDA_BF16}


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need(t: torch.Tensor, name: str, dtype=None, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _prefill_args(q, k, v, gate, gate_shape_tail, beta, h0, cu_seqlens, o, hT,
                  output_final_state, check_gate=True):
    """Check a prefill call's tensors and allocate missing outputs; returns the
    pointer tuple of the C prefill entry points and (o, hT, N, T, H)."""
    if q.dim() != 3 or q.shape[2] != D:
        raise ValueError("q must be [T, H, 128]")
    T, H, _ = q.shape
    dev = q.device
    if q.dtype not in _DT:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, (T, H, D), dev)
    if check_gate:
        _need(gate, "log gate", torch.float32, (T, H) + gate_shape_tail, dev)
    _need(beta, "beta", torch.float32, (T, H), dev)
    if cu_seqlens is None:
        N = 1
    else:
        _need(cu_seqlens, "cu_seqlens", torch.int32, None, dev)
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must be [N+1]")
        N = cu_seqlens.numel() - 1
    if h0 is not None:
        _need(h0, "h0", torch.float32, (N, H, D, D), dev)
    if o is None:
        o = torch.empty_like(q)
    else:
        _need(o, "o", q.dtype, (T, H, D), dev)
    if output_final_state and hT is None:
        hT = torch.empty((N, H, D, D), dtype=torch.float32, device=dev)
    elif hT is not None:
        _need(hT, "hT", torch.float32, (N, H, D, D), dev)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(beta), _ptr(h0), _ptr(cu_seqlens),
            N, T, H, _DT[q.dtype], _ptr(o), _ptr(hT))
    return args, (o, hT, N, T, H)


def dplr_chunk_fwd(q, k, v, a, b, log_alpha, h0=None, cu_seqlens=None, o=None, hT=None,
                   output_final_state: bool = True):
    """General DPLR prefill (comparison kernel): S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} +
    k_t v_t^T. q, k, v, a, b: [T, H, 128] bf16 or fp32 (same dtype); log_alpha: [T, H, 128]
    fp32; h0, cu_seqlens as chunk_fwd. Returns (o, hT)."""
    lib = _native.load()
    for name, t in (("a", a), ("b", b)):
        _need(t, name, q.dtype, tuple(q.shape), q.device)
    T, H, _ = q.shape
    dummy_beta = torch.empty((T, H), dtype=torch.float32, device=q.device)
    args, (o, hT, N, T, H) = _prefill_args(q, k, v, log_alpha, (D,), dummy_beta, h0, cu_seqlens,
                                           o, hT, output_final_state)
    q_, k_, v_, la_, _, h0_, cu_, N_, T_, H_, dt_, o_, hT_ = args
    st = lib.kda_dplr_chunk_fwd(q_, k_, v_, _ptr(a), _ptr(b), la_, h0_, cu_, N_, T_, H_, dt_, o_,
                                hT_, _stream_ptr(q.device))
    _native.check(st, "kda_dplr_chunk_fwd")
    return o, hT


def short_conv_swish(x, w, cu_seqlens=None, y=None):
    """Causal 4-tap depthwise convolution + Swish over tokens, restarted per sequence.

    x: [T, H, 128] (or [T, C]) bf16; w: [C, 4] fp32 with C = H * 128; cu_seqlens:
    [N+1] int32 on the device or None. Returns y like x.
    """
    lib = _native.load()
    dev = x.device
    T = x.shape[0]
    C = x.numel() // max(T, 1) if T else int(torch.tensor(x.shape[1:]).prod())
    _need(x, "x", torch.bfloat16, None, dev)
    _need(w, "w", torch.float32, (C, 4), dev)
    if cu_seqlens is None:
        N = 1
    else:
        _need(cu_seqlens, "cu_seqlens", torch.int32, None, dev)
        N = cu_seqlens.numel() - 1
    if y is None:
        y = torch.empty_like(x)
    else:
        _need(y, "y", torch.bfloat16, tuple(x.shape), dev)
    st = lib.kda_short_conv_swish(_ptr(x), _ptr(w), _ptr(cu_seqlens), N, T, C, _ptr(y),
                                  _stream_ptr(dev))
    _native.check(st, "kda_short_conv_swish")
    return y


def chunk_fwd_fused(q_pre, k_pre, v, decay_pre, beta_pre, gate_pre, norm_w, h0=None,
                    cu_seqlens=None, o=None, hT=None, output_final_state: bool = True,
                    split: bool = True):
    """KDA prefill with the layer's activations and output gate fused in.

    q_pre, k_pre, v, decay_pre, gate_pre: [T, H, 128] bf16; beta_pre: [T, H] fp32;
    norm_w: [128] fp32. q and k are L2-normalised in the kernel, log alpha =
    logsigmoid(decay_pre), beta = sigmoid(beta_pre), and the output is the head-wise
    RMSNorm of o times norm_w times sigmoid(gate_pre). Returns (o_out, hT).
    """
    lib = _native.load()
    T, H, _ = q_pre.shape
    dev = q_pre.device
    _need(q_pre, "q_pre", torch.bfloat16, (T, H, D), dev)
    _need(decay_pre, "decay_pre", torch.bfloat16, (T, H, D), dev)
    _need(gate_pre, "gate_pre", torch.bfloat16, (T, H, D), dev)
    _need(norm_w, "norm_w", torch.float32, (D,), dev)
    args, (o, hT, N, T, H) = _prefill_args(q_pre, k_pre, v, None, None, beta_pre, h0,
                                           cu_seqlens, o, hT, output_final_state,
                                           check_gate=False)
    ws_bytes = 0
    if split:
        ws_bytes = lib.kda_chunk_fwd_workspace_size(N, T, H, _native.KDA_BF16,
                                                    int(cu_seqlens is not None))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    q_, k_, v_, _, b_, h0_, cu_, N_, T_, H_, _, o_, hT_ = args
    st = lib.kda_chunk_fwd_fused(q_, k_, v_, _ptr(decay_pre), b_, _ptr(gate_pre), _ptr(norm_w),
                                 h0_, cu_, N_, T_, H_, o_, hT_, _ptr(ws), ws_bytes, _stream_ptr(dev))
    _native.check(st, "kda_chunk_fwd_fused")
    return o, hT


def gdn_chunk_fwd(q, k, v, log_a, beta, h0=None, cu_seqlens=None, o=None, hT=None,
                  output_final_state: bool = True, split: bool = True):
    """Chunkwise Gated DeltaNet prefill: KDA with one scalar gate per token and head.

    q, k, v: [T, H, 128] bf16 or fp32; log_a: [T, H] fp32 (log of the gate);
    beta: [T, H] fp32; h0, cu_seqlens, o, hT: as chunk_fwd. With ``split`` a single
    long bf16 sequence is split in time over a workspace allocated here.
    """
    lib = _native.load()
    args, (o, hT, N, T, H) = _prefill_args(q, k, v, log_a, (), beta, h0, cu_seqlens, o, hT,
                                           output_final_state)
    ws_bytes = 0
    if split:
        ws_bytes = lib.kda_chunk_fwd_workspace_size(N, T, H, _DT[q.dtype],
                                                    int(cu_seqlens is not None))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device) if ws_bytes else None
    st = lib.kda_gdn_chunk_fwd_ws(*args, _ptr(ws), ws_bytes, _stream_ptr(q.device))
    _native.check(st, "kda_gdn_chunk_fwd_ws")
    return o, hT


def chunk_fwd(q, k, v, log_alpha, beta, h0=None, cu_seqlens=None, o=None, hT=None,
              output_final_state: bool = True, kernel: str = "auto"):
    """Chunkwise KDA prefill.

    q, k, v: [T, H, 128] bf16 or fp32 (same dtype); log_alpha: [T, H, 128] fp32;
    beta: [T, H] fp32; h0: [N, H, 128, 128] fp32 or None; cu_seqlens: [N+1] int32
    on the device or None (one sequence). Returns (o, hT) with o like q and hT
    [N, H, 128, 128] fp32 (None if output_final_state is False).
    ``kernel``: "auto" (tensor cores for bf16, CUDA cores for fp32; a single long
    bf16 sequence is split in time over a workspace allocated here), "static" (as
    "auto", with the library's module-resident scratch instead: no allocation),
    "single" (as "auto" but never split) or "simt" (always the fp32 CUDA-core chunk
    kernel).
    """
    lib = _native.load()
    if q.dim() != 3 or q.shape[2] != D:
        raise ValueError("q must be [T, H, 128]")
    T, H, _ = q.shape
    dev = q.device
    if q.dtype not in _DT:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, (T, H, D), dev)
    _need(log_alpha, "log_alpha", torch.float32, (T, H, D), dev)
    _need(beta, "beta", torch.float32, (T, H), dev)
    if cu_seqlens is None:
        N = 1
    else:
        _need(cu_seqlens, "cu_seqlens", torch.int32, None, dev)
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must be [N+1]")
        N = cu_seqlens.numel() - 1
    if h0 is not None:
        _need(h0, "h0", torch.float32, (N, H, D, D), dev)
    if o is None:
        o = torch.empty_like(q)
    else:
        _need(o, "o", q.dtype, (T, H, D), dev)
    if output_final_state and hT is None:
        hT = torch.empty((N, H, D, D), dtype=torch.float32, device=dev)
    elif hT is not None:
        _need(hT, "hT", torch.float32, (N, H, D, D), dev)
    if kernel not in ("auto", "static", "single", "simt"):
        raise ValueError("kernel must be 'auto', 'static', 'single' or 'simt'")
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(h0), _ptr(cu_seqlens),
            N, T, H, _DT[q.dtype], _ptr(o), _ptr(hT))
    if kernel == "simt":
        st, name = lib.kda_chunk_fwd_simt(*args, _stream_ptr(dev)), "kda_chunk_fwd_simt"
    elif kernel == "static":
        st, name = lib.kda_chunk_fwd_static(*args, _stream_ptr(dev)), "kda_chunk_fwd_static"
    else:
        ws_bytes = 0
        if kernel == "auto":
            ws_bytes = lib.kda_chunk_fwd_workspace_size(N, T, H, _DT[q.dtype],
                                                        int(cu_seqlens is not None))
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
        st = lib.kda_chunk_fwd_ws(*args, _ptr(ws), ws_bytes, _stream_ptr(dev))
        name = "kda_chunk_fwd_ws"
        # (the caching allocator keeps ws alive for the stream's use of it)
    _native.check(st, name)
    return o, hT


def split_plan(n_heads: int, t_total: int, n_sms: int = 0, workspace_bytes: Optional[int] = None):
    """Segment bounds of the time split that kda_chunk_fwd_ws uses for one bf16
    sequence (token offsets, n + 1 of them), or [] when the single pass runs.
    n_sms = 0 plans for the current device; workspace_bytes None = unlimited."""
    import ctypes
    lib = _native.load()
    bounds = (ctypes.c_int64 * (_native.KDA_MAX_SEGMENTS + 1))()
    ws = _native.SIZE_MAX if workspace_bytes is None else int(workspace_bytes)
    n = lib.kda_chunk_fwd_split_plan(int(n_heads), int(t_total), int(n_sms), ws, bounds)
    if n < 0:
        raise KdaError(n, "kda_chunk_fwd_split_plan")
    return [int(bounds[i]) for i in range(n + 1)] if n >= 2 else []


def decode_step(q, k, v, log_alpha, beta, state, o=None):
    """One recurrent KDA step per (sequence, head), state updated in place.

    q, k, v: [N, H, 128] bf16 or fp32; log_alpha: [N, H, 128], beta: [N, H]
    (bf16 or fp32, same dtype); state: [N, H, 128, 128] fp32. Returns o like q.
    """
    lib = _native.load()
    if q.dim() != 3 or q.shape[2] != D:
        raise ValueError("q must be [N, H, 128]")
    N, H, _ = q.shape
    dev = q.device
    if q.dtype not in _DT or log_alpha.dtype not in _DT:
        raise TypeError("unsupported dtype")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, (N, H, D), dev)
    _need(log_alpha, "log_alpha", log_alpha.dtype, (N, H, D), dev)
    _need(beta, "beta", log_alpha.dtype, (N, H), dev)
    _need(state, "state", torch.float32, (N, H, D, D), dev)
    if o is None:
        o = torch.empty_like(q)
    else:
        _need(o, "o", q.dtype, (N, H, D), dev)
    st = lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(state),
                             _ptr(o), N, H, _DT[q.dtype], _DT[log_alpha.dtype], _stream_ptr(dev))
    _native.check(st, "kda_decode_step")
    return o


def decode_tokens(q, k, v, log_alpha, beta, state, o=None):
    """Several recurrent KDA steps per (sequence, head) in one call, state in place.

    q, k, v: [N, t, H, 128] bf16 or fp32 (sequence-major, t = 1..16 new tokens per
    sequence); log_alpha: [N, t, H, 128] and beta: [N, t, H] (bf16 or fp32, same
    dtype); state: [N, H, 128, 128] fp32, read once and written once. Returns o like q.
    """
    lib = _native.load()
    if q.dim() != 4 or q.shape[3] != D:
        raise ValueError("q must be [N, t, H, 128]")
    N, t, H, _ = q.shape
    if not 1 <= t <= _native.KDA_DECODE_MAX_TOKENS:
        raise ValueError(f"t must be in 1..{_native.KDA_DECODE_MAX_TOKENS}")
    dev = q.device
    if q.dtype not in _DT or log_alpha.dtype not in _DT:
        raise TypeError("unsupported dtype")
    for name, x in (("q", q), ("k", k), ("v", v)):
        _need(x, name, q.dtype, (N, t, H, D), dev)
    _need(log_alpha, "log_alpha", log_alpha.dtype, (N, t, H, D), dev)
    _need(beta, "beta", log_alpha.dtype, (N, t, H), dev)
    _need(state, "state", torch.float32, (N, H, D, D), dev)
    if o is None:
        o = torch.empty_like(q)
    else:
        _need(o, "o", q.dtype, (N, t, H, D), dev)
    st = lib.kda_decode_tokens(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                               _ptr(state), _ptr(o), N, t, H, _DT[q.dtype], _DT[log_alpha.dtype],
                               _stream_ptr(dev))
    _native.check(st, "kda_decode_tokens")
    return o


def device_status(device=None) -> int:
    """Read and clear the library's device-side error word (synchronises)."""
    lib = _native.load()
    dev = torch.device("cuda") if device is None else torch.device(device)
    return int(lib.kda_device_status(_stream_ptr(dev)))

"""fp64 reference of the operations around the KDA recurrence (test infrastructure only).

The Kimi Linear pages put these in the layer that produces the operator's inputs and
consumes its output (Kimi Linear summary, section 4 "The Kimi Linear Model
Architecture"; "Kimi Linear -- Forgetting, Channel by Channel", section "Other
Components"; Rationalist Deep-Dive, section 5.3):

  * q, k: short depthwise convolution, Swish, then L2 normalisation per head;
  * v: short depthwise convolution, Swish;
  * the decay: a decay function of a (low-rank) projection;
  * beta: a sigmoid of a projection;
  * the output: head-wise RMSNorm, then a data-dependent sigmoid gate.

Readings where the pages leave a detail open (each is listed with the others in the
repository's design notes):
  * the decay function is log alpha = logsigmoid(x), the function the workloads use to
    draw log alpha, applied per channel to a pre-activation x;
  * L2 normalisation divides by sqrt(sum x^2 + L2_EPS), L2_EPS = 1e-12 (it only guards
    an all-zero row);
  * RMSNorm divides each head's 128 values by sqrt(mean o^2 + RMS_EPS), RMS_EPS = 1e-6,
    and multiplies by a weight of 128 values shared by the heads;
  * the short convolution is causal over the tokens of one sequence: y_t = sum_i
    w[i] x_{t-3+i} with x = 0 before the sequence's first token, one 4-tap filter per
    channel, no bias.

Every function is plain numpy in fp64, written from those definitions one operation
at a time. Nothing here is shared with the CUDA path.
"""

from __future__ import annotations

import numpy as np

L2_EPS = 1e-12
RMS_EPS = 1e-6
CONV_TAPS = 4


def _f64(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu").double().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def sigmoid(x):
    x = _f64(x)
    return 1.0 / (1.0 + np.exp(-x))


def logsigmoid(x):
    """log(sigmoid(x)) = -log(1 + e^{-x}), evaluated without overflow."""
    x = _f64(x)
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


def swish(x):
    x = _f64(x)
    return x * sigmoid(x)


def l2_normalize(x):
    """Each row of the last axis divided by its Euclidean length."""
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + L2_EPS)


def rms_norm(o, weight):
    """Head-wise RMSNorm over the last axis, times a per-channel weight."""
    o = _f64(o)
    w = _f64(weight)
    return o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + RMS_EPS) * w


def output_gate(o, weight, gate_pre):
    """RMSNorm of the recurrence's output, then the sigmoid gate."""
    return rms_norm(o, weight) * sigmoid(gate_pre)


def short_conv(x, w, cu_seqlens=None):
    """Causal depthwise convolution over tokens, restarted at every sequence.

    x: [T, C] (any trailing shape flattened into C by the caller); w: [C, 4] (tap i
    multiplies the input i - 3 tokens away, tap 3 the current one);
    cu_seqlens: [N+1] or None (one sequence). Returns [T, C] fp64.
    """
    x = _f64(x)
    w = _f64(w)
    T = x.shape[0]
    cu = [0, T] if cu_seqlens is None else [int(c) for c in _f64(cu_seqlens)]
    y = np.zeros_like(x)
    for n in range(len(cu) - 1):
        a, b = cu[n], cu[n + 1]
        for t in range(a, b):
            for i in range(CONV_TAPS):
                s = t - (CONV_TAPS - 1) + i
                if s >= a:
                    y[t] += w[:, i] * x[s]
    return y


def short_conv_swish(x, w, cu_seqlens=None):
    return swish(short_conv(x, w, cu_seqlens))


def fused_layer_forward(q_pre, k_pre, v_pre, decay_pre, beta_pre, gate_pre, norm_weight,
                        h0=None, cu_seqlens=None, conv_w=None, n_threads: int = 0,
                        col_block: int = 0, return_pre_norm: bool = False):
    """The recurrence with the operations around it, in the order the pages give.

    q_pre, k_pre, v_pre: [T, H, 128] (the projections' outputs); decay_pre: [T, H, 128]
    (log alpha = logsigmoid(decay_pre)); beta_pre: [T, H] (beta = sigmoid(beta_pre));
    gate_pre: [T, H, 128]; norm_weight: [128]; conv_w: None, or a dict with "q", "k", "v"
    filters [H * 128, 4] (short convolution + Swish before the rest). Returns
    (o_final [T, H, 128], hT [N, H, 128, 128]) in fp64, and with return_pre_norm also
    the recurrence's output o before the RMSNorm.

    The recurrence itself is the C oracle (kda_oracle.c), which reads its inputs as
    fp32: the fp64 results of the steps before it are rounded to fp32 there (a relative
    change of at most 2^-24, far below any tolerance used with this function).
    """
    from .kda_oracle import oracle_forward
    q, k, v = _f64(q_pre), _f64(k_pre), _f64(v_pre)
    T, H, d = q.shape
    if conv_w is not None:
        cu = None if cu_seqlens is None else _f64(cu_seqlens)
        q = short_conv_swish(q.reshape(T, H * d), conv_w["q"], cu).reshape(T, H, d)
        k = short_conv_swish(k.reshape(T, H * d), conv_w["k"], cu).reshape(T, H, d)
        v = short_conv_swish(v.reshape(T, H * d), conv_w["v"], cu).reshape(T, H, d)
    q = l2_normalize(q)
    k = l2_normalize(k)
    log_alpha = logsigmoid(decay_pre)
    beta = sigmoid(beta_pre)
    o, hT = oracle_forward(q, k, v, log_alpha, beta, h0=h0, cu_seqlens=cu_seqlens,
                           n_threads=n_threads, col_block=col_block)
    if return_pre_norm:
        return output_gate(o, norm_weight, gate_pre), hT, o
    return output_gate(o, norm_weight, gate_pre), hT

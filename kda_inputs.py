"""Seeded synthetic inputs for KDA, shared by the tests, the benchmark and the oracle runs.

This module only draws random numbers and shapes them. It holds none of the
recurrence's arithmetic: the activations applied here (L2 normalisation of q and
k, sigmoid for beta, logsigmoid for the log-decay) are how the Kimi Linear
summary describes the layer *producing* the operator's inputs (section 4 "The
Kimi Linear Model Architecture": q and k normalised to unit length; beta from a
sigmoid; the decay from a low-rank projection and a decay function). Trained
weights are not available, so the pre-activations are Gaussian draws.

Recipe (the workloads are shaped like the 48B model's KDA layers: 32 heads,
head dim 128):
  * q, k ~ N(0, 1), then L2-normalised per (token, head) in fp32, then rounded
    to the storage dtype (so normalisation is exact only up to that rounding);
  * v ~ N(0, 1);
  * beta = sigmoid(N(0, 1));
  * log_alpha = logsigmoid(x), x ~ N(mu, 1) drawn per (token, head, channel),
    computed in fp32 (mu = 3 normally, 4 for the long-context workload);
  * h0 ~ N(0, 0.02) (standard deviation 0.02) where the workload has one.
Storage dtypes follow each workload: q/k/v bf16 (fp32 for the tiny case); gates
fp32 for prefill and bf16 for decode; state fp32.

Large workloads are drawn on the device in token slabs to bound peak memory.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch

D = 128  # head dimension d_k = d_v


@dataclasses.dataclass(frozen=True)
class PrefillConfig:
    name: str
    lens: tuple            # per-sequence token counts (None -> drawn, see varlen)
    n_heads: int
    qkv_dtype: torch.dtype
    x_mean: float          # mean of the logsigmoid pre-activation
    h0: bool               # random initial state per sequence
    seed: int
    varlen: Optional[tuple] = None  # (n_seqs, lo, hi): lengths ~ U[lo, hi] from the seed


# The five workloads (prefill 0-3 and decode 4). Sizes are fixed; seeds = index.
PREFILL_CONFIGS = {
    0: PrefillConfig("tiny_fp32_T256_H2", (256,), 2, torch.float32, 3.0, False, 0),
    1: PrefillConfig("prefill_bf16_T4096_H32", (4096,), 32, torch.bfloat16, 3.0, True, 1),
    2: PrefillConfig("varlen16_bf16_H32", None, 32, torch.bfloat16, 3.0, True, 2,
                     varlen=(16, 512, 8192)),
    3: PrefillConfig("longctx_bf16_T1048576_H32", (1048576,), 32, torch.bfloat16, 4.0, False, 3),
}


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    n_seqs: int
    n_heads: int
    steps: int
    qkv_dtype: torch.dtype
    gate_dtype: torch.dtype
    x_mean: float
    state_std: float
    seed: int


DECODE_CONFIG = DecodeConfig("decode_bf16_N256_H32", 256, 32, 1000, torch.bfloat16,
                             torch.bfloat16, 3.0, 0.02, 4)


def varlen_lengths(n_seqs: int, lo: int, hi: int, seed: int) -> list:
    g = torch.Generator(device="cpu").manual_seed(1000 + seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n_seqs,), generator=g)]


def config_lengths(cfg: PrefillConfig) -> list:
    if cfg.varlen is not None:
        return varlen_lengths(*cfg.varlen, seed=cfg.seed)
    return list(cfg.lens)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    # per-(token, head) L2 normalisation of the last axis, in fp32
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def make_prefill(lens, n_heads: int, qkv_dtype=torch.bfloat16, gate_dtype=torch.float32,
                 x_mean: float = 3.0, h0: bool = False, seed: int = 0, device="cpu",
                 slab: int = 1 << 16, d: int = D, h0_std: float = 0.02,
                 scalar_gate: bool = False):
    """Draw a packed prefill batch.

    Returns a dict with q, k, v [T, H, d] (qkv_dtype), log_alpha [T, H, d] and
    beta [T, H] (gate_dtype), h0 [N, H, d, d] fp32 or None, cu_seqlens [N+1] int32
    and lens (list). With scalar_gate the log-decay is one value per token and head,
    log_alpha [T, H] (the Gated DeltaNet gate), drawn the same way.
    """
    lens = [int(x) for x in lens]
    T = sum(lens)
    N = len(lens)
    g = _gen(device, seed)
    q = torch.empty((T, n_heads, d), dtype=qkv_dtype, device=device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    la = torch.empty((T, n_heads) if scalar_gate else (T, n_heads, d), dtype=gate_dtype,
                     device=device)
    b = torch.empty((T, n_heads), dtype=gate_dtype, device=device)
    for t0 in range(0, T, slab):
        t1 = min(T, t0 + slab)
        shp = (t1 - t0, n_heads, d)
        q[t0:t1] = _unit_rows(torch.randn(shp, generator=g, device=device)).to(qkv_dtype)
        k[t0:t1] = _unit_rows(torch.randn(shp, generator=g, device=device)).to(qkv_dtype)
        v[t0:t1] = torch.randn(shp, generator=g, device=device).to(qkv_dtype)
        x = torch.randn(shp[:2] if scalar_gate else shp, generator=g, device=device) + x_mean
        la[t0:t1] = torch.nn.functional.logsigmoid(x).to(gate_dtype)
        b[t0:t1] = torch.sigmoid(torch.randn(shp[:2], generator=g, device=device)).to(gate_dtype)
    h0_t = None
    if h0:
        h0_t = (torch.randn((N, n_heads, d, d), generator=g, device=device) * h0_std).float()
    cu = torch.zeros(N + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(torch.int32)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=b, h0=h0_t, cu_seqlens=cu.to(device),
                lens=lens)


def make_config(idx: int, device="cpu", lens_override=None, heads_override=None):
    cfg = PREFILL_CONFIGS[idx]
    lens = lens_override if lens_override is not None else config_lengths(cfg)
    H = heads_override if heads_override is not None else cfg.n_heads
    return make_prefill(lens, H, cfg.qkv_dtype, torch.float32, cfg.x_mean, cfg.h0, cfg.seed,
                        device)


def make_decode(n_seqs: int, n_heads: int, steps: int, qkv_dtype=torch.bfloat16,
                gate_dtype=torch.bfloat16, x_mean: float = 3.0, state_std: float = 0.02,
                seed: int = 4, device="cpu", d: int = D):
    """Draw decode inputs: step-major q, k, v, log_alpha [steps, N, H, d], beta
    [steps, N, H], plus the starting state [N, H, d, d] fp32 ~ N(0, state_std)."""
    g = _gen(device, seed)
    state = (torch.randn((n_seqs, n_heads, d, d), generator=g, device=device) * state_std).float()
    shp = (steps, n_seqs, n_heads, d)
    q = torch.empty(shp, dtype=qkv_dtype, device=device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    la = torch.empty(shp, dtype=gate_dtype, device=device)
    b = torch.empty(shp[:3], dtype=gate_dtype, device=device)
    for s in range(steps):
        q[s] = _unit_rows(torch.randn(shp[1:], generator=g, device=device)).to(qkv_dtype)
        k[s] = _unit_rows(torch.randn(shp[1:], generator=g, device=device)).to(qkv_dtype)
        v[s] = torch.randn(shp[1:], generator=g, device=device).to(qkv_dtype)
        x = torch.randn(shp[1:], generator=g, device=device) + x_mean
        la[s] = torch.nn.functional.logsigmoid(x).to(gate_dtype)
        b[s] = torch.sigmoid(torch.randn(shp[1:3], generator=g, device=device)).to(gate_dtype)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=b, state=state)


def make_decode_config(device="cpu", n_seqs=None, steps=None):
    c = DECODE_CONFIG
    return make_decode(n_seqs or c.n_seqs, c.n_heads, steps or c.steps, c.qkv_dtype,
                       c.gate_dtype, c.x_mean, c.state_std, c.seed, device)


def make_parallel_keys(T: int, n_heads: int, qkv_dtype=torch.bfloat16, eps: float = 1e-2,
                       run: int = 16, beta_lo: float = 0.98, x_mean: float = 8.0,
                       h0_std: float = 1.0, seed: int = 0, device="cpu", d: int = D):
    """A hard case for the chunk form's triangular solve: one sequence whose keys come
    in runs of `run` nearly parallel unit vectors (k_t = normalise(k_base + eps * n_t),
    a new base direction per run), erase strengths beta ~ U[beta_lo, 1], decay close to
    one (log_alpha = logsigmoid(x), x ~ N(x_mean, 1)) and a large initial state
    (h0 ~ N(0, h0_std)). q and v are drawn as in make_prefill. Same dict as make_prefill.
    """
    g = _gen(device, seed)
    shp = (T, n_heads, d)
    q = _unit_rows(torch.randn(shp, generator=g, device=device)).to(qkv_dtype)
    n_runs = (T + run - 1) // run
    base = torch.randn((n_runs, n_heads, d), generator=g, device=device)
    base = base.repeat_interleave(run, dim=0)[:T]
    k = _unit_rows(_unit_rows(base) + eps * torch.randn(shp, generator=g, device=device))
    k = k.to(qkv_dtype)
    v = torch.randn(shp, generator=g, device=device).to(qkv_dtype)
    x = torch.randn(shp, generator=g, device=device) + x_mean
    la = torch.nn.functional.logsigmoid(x).float()
    b = (beta_lo + (1.0 - beta_lo) * torch.rand((T, n_heads), generator=g, device=device)).float()
    h0_t = (torch.randn((1, n_heads, d, d), generator=g, device=device) * h0_std).float()
    cu = torch.tensor([0, T], dtype=torch.int32, device=device)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=b, h0=h0_t, cu_seqlens=cu, lens=[T])


def make_fused_prefill(lens, n_heads: int, x_mean: float = 3.0, h0: bool = True, seed: int = 0,
                       device="cpu", d: int = D, h0_std: float = 0.02):
    """Inputs of the fused entry point: the producing layer's raw outputs.

    q_pre, k_pre, v ~ N(0, 1) bf16 (q and k not normalised); decay_pre ~ N(x_mean, 1)
    bf16 (the decay pre-activation); beta_pre ~ N(0, 1) fp32; gate_pre ~ N(0, 1) bf16
    (the output gate pre-activation); norm_w ~ U(0.5, 1.5) fp32 [d]; h0 ~ N(0, h0_std).
    """
    lens = [int(x) for x in lens]
    T, N = sum(lens), len(lens)
    g = _gen(device, seed)
    shp = (T, n_heads, d)
    bf = torch.bfloat16
    out = dict(
        q_pre=torch.randn(shp, generator=g, device=device).to(bf),
        k_pre=torch.randn(shp, generator=g, device=device).to(bf),
        v=torch.randn(shp, generator=g, device=device).to(bf),
        decay_pre=(torch.randn(shp, generator=g, device=device) + x_mean).to(bf),
        beta_pre=torch.randn((T, n_heads), generator=g, device=device).float(),
        gate_pre=torch.randn(shp, generator=g, device=device).to(bf),
        norm_w=(0.5 + torch.rand((d,), generator=g, device=device)).float(),
    )
    out["h0"] = ((torch.randn((N, n_heads, d, d), generator=g, device=device) * h0_std).float()
                 if h0 else None)
    cu = torch.zeros(N + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(torch.int32)
    out["cu_seqlens"] = cu.to(device)
    out["lens"] = lens
    return out


def make_dplr_prefill(lens, n_heads: int, qkv_dtype=torch.bfloat16, x_mean: float = 3.0,
                      h0: bool = True, seed: int = 0, device="cpu", d: int = D,
                      h0_std: float = 0.02):
    """Inputs of the general DPLR recurrence: those of make_prefill plus free low-rank
    factors a = beta u and b = w * alpha, with u and w unit vectors drawn independently
    of k (KDA would take u = w = k). Returns make_prefill's dict plus a and b."""
    inp = make_prefill(lens, n_heads, qkv_dtype, torch.float32, x_mean, h0, seed, device,
                       d=d, h0_std=h0_std)
    g = _gen(device, seed + 7777)
    T = sum(int(x) for x in lens)
    shp = (T, n_heads, d)
    u = _unit_rows(torch.randn(shp, generator=g, device=device))
    w = _unit_rows(torch.randn(shp, generator=g, device=device))
    inp["a"] = (inp["beta"][:, :, None] * u).to(qkv_dtype)
    inp["b"] = (w * torch.exp(inp["log_alpha"])).to(qkv_dtype)
    return inp

"""Benchmark: KDA prefill tokens/s (H=32, d=128) and decode-step HBM GB/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0. A "step" is one pass of the hot path over one batch:
one chunkwise prefill launch over the long-context workload (1,048,576 tokens,
32 heads, bf16 q/k/v, fp32 gates) -- the headline `value` -- and the decode
step on its own workload (256 sequences x 32 heads, fp32 state) timed
separately and reported under "decode".

Multi-GPU: every rank processes its own independent batch (replicas, no
collective on the data path); value = all ranks' tokens / max-over-ranks time.
`--impl reference` times the fp64 oracle on the host cores instead.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import kda_inputs  # noqa: E402

METRIC = "KDA prefill tokens/s (H=32,d=128) & decode-step HBM GB/s vs peak, 1xB200"
WORKLOADS = {"longctx": 3, "prefill4k": 1, "varlen16": 2}
D = 128
PREFILL_BYTES_PER_TOKEN_HEAD = 3 * 2 * D + 4 * D + 4 + 2 * D   # q,k,v bf16 + log_alpha f32 + beta + o
STATE_BYTES = 4 * D * D
DECODE_BYTES_PER_CHAIN = 2 * STATE_BYTES + 4 * 2 * D + 2 + 2 * D   # state rw + q,k,v,la + beta + o
DECODE_TOKENS = 4   # tokens per sequence per call of the multi-token decode step


def decode_tokens_bytes_per_chain(t: int) -> int:
    """State read + write once, plus q, k, v, log_alpha, beta and o of t tokens (bf16)."""
    return 2 * STATE_BYTES + t * (4 * 2 * D + 2 + 2 * D)
L2_BYTES = 126 * 1024 * 1024


# The sources that make up the profiled prefill path: the chunk kernel, its sm_100a
# building blocks, the segment scan, and the file that builds its tensor maps and
# launches it (plus the ABI header). The decode and fp32 kernels live in files of
# their own and do not enter.
CHUNK_KERNEL_SOURCES = ("kda_api.cu", "kda_chunk_tc.cuh", "kda_common.cuh", "kda_segment.cuh",
                        "kda_sm100.cuh")


def _source_hash() -> str:
    """sha256 prefix of the prefill chunk kernel's sources (CHUNK_KERNEL_SOURCES and
    include/kda.h): the ncu figures in profiles/ hold while it is unchanged."""
    import hashlib
    csrc = os.path.join(ROOT, "channel_wise_gated_b200", "csrc")
    files = [os.path.join(csrc, f) for f in sorted(CHUNK_KERNEL_SOURCES)]
    files.append(os.path.join(ROOT, "include", "kda.h"))
    h = hashlib.sha256()
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _profiled_traffic(split: bool, token_heads: int):
    """DRAM bytes of one long-context prefill call from the committed one-pass ncu capture
    (profiles/kda_chunk_tc_longctx_dram.md), or None when the kernel sources changed since
    that capture or the call is not the one it describes."""
    import re
    path = os.path.join(ROOT, "profiles", "kda_chunk_tc_longctx_dram.md")
    if not split or token_heads != 32 * 1048576 or not os.path.exists(path):
        return None
    txt = open(path).read()
    mh = re.search(r"^source_hash: ([0-9a-f]+)$", txt, re.M)
    mb = re.search(r"^longctx_call_dram_bytes: ([0-9.]+)$", txt, re.M)
    if not mh or not mb or mh.group(1) != _source_hash():
        return None
    return float(mb.group(1))


def _profiled_metric(name: str):
    """A figure recorded with the ncu capture summarised in
    profiles/kda_chunk_tc_prefill4k_full.md, or None when the kernel sources changed
    since that capture."""
    import re
    path = os.path.join(ROOT, "profiles", "kda_chunk_tc_prefill4k_full.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    mh = re.search(r"^source_hash: ([0-9a-f]+)$", txt, re.M)
    mv = re.search(rf"^{name}: ([0-9.]+)$", txt, re.M)
    if not mh or not mv or mh.group(1) != _source_hash():
        return None
    return float(mv.group(1))


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while a region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="kda_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return ws, rank, local


def _barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def _reduce_device() -> str:
    # NCCL reduces device tensors; gloo (the CPU test backend) host tensors
    return "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"


def _max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def _sum_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def replica_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch (replicas): seeds are distinct per rank."""
    return base_seed + 100 * rank


def replica_throughput(units: float, ms: float, ws: int) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return _sum_over_ranks(units, ws) / (_max_over_ranks(ms, ws) / 1e3)


def _oracle_sample_rate(cfg_idx: int, target_s: float, seed_heads=(0, 1), max_tokens=1 << 20):
    """Time the fp64 oracle on a bounded sample of a prefill workload.

    Returns (tokens/s scaled to the workload's head count, sample description,
    threads used, seconds). Throughput scales linearly in heads (heads are
    independent), so token-heads/s over the sampled heads / n_heads is the
    oracle's tokens/s for the full head count.
    """
    import oracle
    cfg = kda_inputs.PREFILL_CONFIGS[cfg_idx]
    H = len(seed_heads)
    threads = oracle.oracle_threads()

    def run(T):
        inp = kda_inputs.make_prefill([T], H, cfg.qkv_dtype, torch.float32, cfg.x_mean, cfg.h0,
                                      cfg.seed, "cpu")
        t0 = time.perf_counter()
        oracle.oracle_forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                              h0=inp["h0"], col_block=max(1, D * H // threads))
        return time.perf_counter() - t0

    T = 2048
    dt = run(T)
    T = int(min(max_tokens, max(2048, T * target_s / max(dt, 1e-3))))
    dt = run(T)
    rate = T * H / dt / cfg.n_heads
    desc = (f"{cfg.name}: first {T} tokens of {H} heads (fp64 oracle, {threads} threads), "
            f"token-heads/s divided by {cfg.n_heads} heads")
    return rate, desc, threads, dt, T


def run_reference(args):
    """The fp64 oracle on the host cores (rank 0 only)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    cfg = kda_inputs.PREFILL_CONFIGS[3]
    threads = oracle.oracle_threads()
    H = 2
    # calibrate a sample of ~4 s per step
    _, _, _, _, T = _oracle_sample_rate(3, 4.0)
    inp = kda_inputs.make_prefill([T], H, cfg.qkv_dtype, torch.float32, cfg.x_mean, cfg.h0,
                                  cfg.seed, "cpu")

    def step():
        oracle.oracle_forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                              col_block=max(1, D * H // threads))

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    rate = args.steps * T * H / dt / cfg.n_heads
    sample = (f"{cfg.name}: first {T} tokens of {H} heads per step (fp64 oracle), "
              f"token-heads/s divided by {cfg.n_heads} heads")
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "T": 1048576, "H": 32, "d": D, "chunk": 64,
                   "sampled_T": T, "sampled_heads": H},
        "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def time_prefill(kda, inp, steps, warmup, ws, stream):
    cu = None if len(inp["lens"]) == 1 else inp["cu_seqlens"]   # one sequence: no cu_seqlens
    fwd = lambda: kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                h0=inp["h0"], cu_seqlens=cu, o=inp["o"], hT=inp["hT"])
    for _ in range(warmup):
        fwd()
    torch.cuda.synchronize()
    _barrier(ws)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for a, b in ev:
        a.record(stream)
        fwd()
        b.record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    _barrier(ws)
    total_ms = t_start.elapsed_time(t_end)
    per_launch = [a.elapsed_time(b) for a, b in ev]
    return total_ms, per_launch


def time_decode(kda, dec, steps, warmup, stream):
    n_avail = dec["q"].shape[0]
    st = dec["state"]
    o = torch.empty_like(dec["q"][0])

    def step(s):
        s = s % n_avail
        kda.decode_step(dec["q"][s], dec["k"][s], dec["v"][s], dec["log_alpha"][s],
                        dec["beta"][s], st, o=o)

    for s in range(warmup):
        step(s)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for s in range(steps):
        step(s)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def time_decode_tokens(kda, pool, state, calls, warmup, stream):
    """kda_decode_tokens calls over a pool of distinct [N, t, H, 128] input sets; the
    state is updated in place by every call."""
    n_avail = len(pool)
    o = torch.empty_like(pool[0]["q"])

    def call(c):
        x = pool[c % n_avail]
        kda.decode_tokens(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state, o=o)

    for c in range(warmup):
        call(c)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for c in range(calls):
        call(c)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def _time_calls(fn, reps, warmup, stream):
    """Average CUDA-event time of `reps` back-to-back calls on `stream`, after warm-up."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def _frac(nbytes, ms, peak_gbs):
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"GBps": gbs, "frac": gbs / peak_gbs, "frac_nominal_8tbs": gbs / 8000.0,
            "algorithmic_bytes": nbytes}


def run_extras(kda, hbm_peak, stream, headline):
    """The other entry points and workloads, each timed on its own (N = 1): the
    contract's single-pass call at the headline size, the T=4096 and packed-batch
    prefills, the Gated DeltaNet and fused-layer variants at the headline size, the
    short convolution, and the general-DPLR comparison (16 heads, batch 1). Inputs are
    drawn on the device before each entry's timed region and larger than L2 where the
    entry is an HBM-bound pass."""
    ex = {}
    D_ = D
    # (1) the contract's entry point (single pass, no workspace) on the headline input
    inp = headline
    T, H = inp["q"].shape[0], inp["q"].shape[1]
    ms = _time_calls(lambda: kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                           inp["beta"], o=inp["o"], hT=inp["hT"],
                                           kernel="single"), 2, 1, stream)
    nbytes = T * H * PREFILL_BYTES_PER_TOKEN_HEAD + H * STATE_BYTES
    ex["contract_single_pass"] = {"entry": "kda_chunk_fwd", "workload": "longctx_bf16_T1048576_H32",
                                  "ms": ms, "tokens_per_s": T / (ms / 1e3),
                                  **_frac(nbytes, ms, hbm_peak)}
    # (2) the smaller prefill workloads, through the workspace entry point
    for key, idx in (("prefill4k", 1), ("varlen16", 2)):
        cfg = kda_inputs.PREFILL_CONFIGS[idx]
        lens = kda_inputs.config_lengths(cfg)
        x = kda_inputs.make_prefill(lens, cfg.n_heads, cfg.qkv_dtype, torch.float32, cfg.x_mean,
                                    cfg.h0, cfg.seed, "cuda")
        cu = None if len(lens) == 1 else x["cu_seqlens"]
        ms = _time_calls(lambda: kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                               h0=x["h0"], cu_seqlens=cu), 20, 3, stream)
        Tt, N = sum(lens), len(lens)
        nbytes = Tt * cfg.n_heads * PREFILL_BYTES_PER_TOKEN_HEAD + 2 * N * cfg.n_heads * STATE_BYTES
        ex[key] = {"entry": "kda_chunk_fwd_ws", "workload": cfg.name, "ms": ms,
                   "tokens_per_s": Tt / (ms / 1e3), **_frac(nbytes, ms, hbm_peak)}
        del x
    torch.cuda.empty_cache()
    return ex


def run_extras_large(kda, hbm_peak, stream, ex):
    """Entries whose inputs are as large as the headline's (run after it is freed)."""
    cfg = kda_inputs.PREFILL_CONFIGS[3]
    T, H = cfg.lens[0], cfg.n_heads
    # (3) Gated DeltaNet: one gate per token and head (4 B instead of 512)
    x = kda_inputs.make_prefill([T], H, cfg.qkv_dtype, torch.float32, cfg.x_mean, cfg.h0,
                                cfg.seed, "cuda", scalar_gate=True)
    o = torch.empty_like(x["q"])
    hT = torch.empty((1, H, D, D), dtype=torch.float32, device="cuda")
    ms = _time_calls(lambda: kda.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                               o=o, hT=hT), 5, 3, stream)
    per_th = 3 * 2 * D + 4 + 4 + 2 * D
    ex["gdn_scalar_gate"] = {"entry": "kda_gdn_chunk_fwd_ws", "workload": f"{cfg.name}_scalar_gate",
                             "ms": ms, "tokens_per_s": T / (ms / 1e3),
                             "bytes_per_token_head": per_th,
                             **_frac(T * H * per_th + H * STATE_BYTES, ms, hbm_peak)}
    del x, o, hT
    torch.cuda.empty_cache()
    # (4) the fused layer path: L2 norm, logsigmoid, sigmoid in the loader, RMSNorm and
    #     gate in the epilogue (bf16 decay 256 B, gate 256 B per token-head)
    x = kda_inputs.make_fused_prefill([T], H, x_mean=cfg.x_mean, h0=False, seed=cfg.seed,
                                      device="cuda")
    o = torch.empty_like(x["q_pre"])
    hT = torch.empty((1, H, D, D), dtype=torch.float32, device="cuda")
    ms = _time_calls(lambda: kda.chunk_fwd_fused(x["q_pre"], x["k_pre"], x["v"], x["decay_pre"],
                                                 x["beta_pre"], x["gate_pre"], x["norm_w"],
                                                 o=o, hT=hT), 5, 3, stream)
    per_th = 3 * 2 * D + 2 * D + 4 + 2 * D + 2 * D   # q k v, decay, beta, gate, o
    ex["fused_layer"] = {"entry": "kda_chunk_fwd_fused", "workload": f"{cfg.name}_fused",
                         "ms": ms, "tokens_per_s": T / (ms / 1e3),
                         "bytes_per_token_head": per_th,
                         "unfused_passes_bytes_per_token_head": (
                             PREFILL_BYTES_PER_TOKEN_HEAD   # the operator itself (fp32 log alpha)
                             + 4 * 2 * D                    # L2 norm of q, k: read + write
                             + 2 * D + 4 * D                # decay activation: read bf16, write fp32
                             + 3 * 2 * D),                  # RMSNorm + gate: read o, gate; write
                         **_frac(T * H * per_th + H * STATE_BYTES, ms, hbm_peak)}
    # (5) the short convolution + Swish of one of q, k, v at the same size
    C = H * D
    wc = (torch.randn((C, 4), device="cuda") * 0.5).float()
    xin = x["q_pre"].reshape(T, C)
    y = torch.empty_like(xin)
    ms = _time_calls(lambda: kda.short_conv_swish(xin, wc, y=y), 5, 3, stream)
    ex["short_conv_swish"] = {"entry": "kda_short_conv_swish", "workload": f"T{T}_C{C}_bf16",
                              "ms": ms, "tokens_per_s": T / (ms / 1e3),
                              **_frac(T * C * 2 * 2, ms, hbm_peak)}
    del x, o, hT, xin, y
    torch.cuda.empty_cache()
    # (6) general DPLR against KDA, the same CUDA-core style, 16 heads, batch 1
    rows = []
    for Tc in (2048, 8192, 65536):
        x = kda_inputs.make_dplr_prefill([Tc], 16, torch.bfloat16, seed=1, device="cuda")
        t_k = _time_calls(lambda: kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                                h0=x["h0"], kernel="simt"), 2, 1, stream)
        t_d = _time_calls(lambda: kda.dplr_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b"],
                                                     x["log_alpha"], h0=x["h0"]), 2, 1, stream)
        t_tc = _time_calls(lambda: kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"],
                                                 x["beta"], h0=x["h0"]), 5, 2, stream)
        rows.append({"T": Tc, "H": 16, "kda_cuda_core_ms": t_k, "dplr_cuda_core_ms": t_d,
                     "dplr_over_kda": t_d / t_k, "kda_tensor_core_ms": t_tc})
        del x
    torch.cuda.empty_cache()
    ex["dplr_comparison"] = {"entries": ["kda_chunk_fwd_simt", "kda_dplr_chunk_fwd",
                                         "kda_chunk_fwd_ws"], "rows": rows}
    return ex


def time_e2e(kda, inp, steps, stream):
    """Public API with host buffers: H2D of the step's inputs from pinned memory,
    the prefill, and D2H of its outputs (o and the final state), every step."""
    names = ["q", "k", "v", "log_alpha", "beta"]
    host = {n: torch.empty(inp[n].shape, dtype=inp[n].dtype, pin_memory=True) for n in names}
    for n in names:
        host[n].copy_(inp[n])
    o_host = torch.empty(inp["o"].shape, dtype=inp["o"].dtype, pin_memory=True)
    h_host = torch.empty(inp["hT"].shape, dtype=inp["hT"].dtype, pin_memory=True)
    dev = {n: torch.empty_like(inp[n]) for n in names}
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = o_host.numel() * o_host.element_size() + h_host.numel() * h_host.element_size()

    cu = None if len(inp["lens"]) == 1 else inp["cu_seqlens"]

    def step():
        for n in names:
            dev[n].copy_(host[n], non_blocking=True)
        o, hT = kda.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                              h0=None, cu_seqlens=cu, o=inp["o"], hT=inp["hT"])
        o_host.copy_(o, non_blocking=True)
        h_host.copy_(hT, non_blocking=True)

    step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    del host, dev, o_host, h_host
    return ms, h2d, d2h


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other entry points' entries (timed after the headline)")
    ap.add_argument("--workload", default="longctx",
                    choices=sorted(WORKLOADS),
                    help="prefill workload (the headline is longctx; prefill4k is the small "
                         "case used for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    ws, rank, local = _dist()
    import channel_wise_gated_b200 as kda
    kda._native.load()   # the in-tree library; raises if missing
    stream = torch.cuda.current_stream()
    hbm_peak, bf16_peak, peak_kind = _peaks()

    # ---- prefill workload (each rank its own batch)
    cfg = kda_inputs.PREFILL_CONFIGS[WORKLOADS[args.workload]]
    lens = kda_inputs.config_lengths(cfg)
    inp = kda_inputs.make_prefill(lens, cfg.n_heads, cfg.qkv_dtype, torch.float32, cfg.x_mean,
                                  cfg.h0, replica_seed(cfg.seed, rank), "cuda")
    T, H = sum(lens), cfg.n_heads
    N = len(lens)
    inp["o"] = torch.empty_like(inp["q"])
    inp["hT"] = torch.empty((N, H, D, D), dtype=torch.float32, device="cuda")
    step_bytes = T * H * PREFILL_BYTES_PER_TOKEN_HEAD + N * H * STATE_BYTES * (
        2 if inp["h0"] is not None else 1)
    # one prefill call = one launch of the chunk kernel, or, for one long sequence
    # split in time, its zero-state pass + the segment scan (3 segments or more) + its
    # correction pass
    n_seg = len(kda.split_plan(H, T)) - 1 if N == 1 else 0
    split = n_seg >= 2
    launches_per_call = (3 if n_seg >= 3 else 2) if split else 1

    with ClockSampler(local) as clk:
        total_ms, per_launch = time_prefill(kda, inp, args.steps, args.warmup, ws, stream)
    clocks = clk.summary()
    max_ms = _max_over_ranks(total_ms, ws)
    value = replica_throughput(float(T * args.steps), total_ms, ws)
    avg_launch_ms = sum(per_launch) / len(per_launch)
    achieved = step_bytes / (avg_launch_ms / 1e3) / 1e9

    # ---- decode workload
    dcfg = kda_inputs.DECODE_CONFIG
    n_pool = 50   # distinct per-step inputs cycled through (all > L2 with the state)
    dec = kda_inputs.make_decode(dcfg.n_seqs, dcfg.n_heads, n_pool, dcfg.qkv_dtype,
                                 dcfg.gate_dtype, dcfg.x_mean, dcfg.state_std,
                                 replica_seed(dcfg.seed, rank), "cuda")
    _barrier(ws)
    dec_ms = _max_over_ranks(time_decode(kda, dec, args.decode_steps, args.warmup, stream), ws)
    chains = dcfg.n_seqs * dcfg.n_heads
    dec_step_us = dec_ms / args.decode_steps * 1e3
    # whole-job bytes per step (every replica moves its own states) over the slowest rank
    dec_gbs = replica_throughput(float(chains * DECODE_BYTES_PER_CHAIN * args.decode_steps),
                                 dec_ms, ws) / 1e9
    # multi-token decode: DECODE_TOKENS consecutive steps of every sequence per call,
    # inputs grouped from the same draws (sequence-major), the same state in place
    t_dec = DECODE_TOKENS
    pool = [{n: dec[n][i * t_dec:(i + 1) * t_dec].transpose(0, 1).contiguous()
             for n in ("q", "k", "v", "log_alpha", "beta")} for i in range(n_pool // t_dec)]
    dt_calls = max(1, args.decode_steps // t_dec)
    _barrier(ws)
    dt_ms = _max_over_ranks(time_decode_tokens(kda, pool, dec["state"], dt_calls, args.warmup,
                                               stream), ws)
    dt_bytes = chains * decode_tokens_bytes_per_chain(t_dec)
    dt_gbs = replica_throughput(float(dt_bytes * dt_calls), dt_ms, ws) / 1e9
    dt_tok_s = replica_throughput(float(dcfg.n_seqs * t_dec * dt_calls), dt_ms, ws)
    del dec, pool
    torch.cuda.empty_cache()

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        ms, h2d, d2h = time_e2e(kda, inp, args.e2e_steps, stream)
        e2e = {"value": replica_throughput(float(T * args.e2e_steps), ms, ws),
               "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": args.e2e_steps}

    extras = None
    if ws == 1 and not args.no_extras and args.workload == "longctx":
        extras = run_extras(kda, hbm_peak, stream, inp)
    del inp
    torch.cuda.empty_cache()
    if extras is not None:
        extras = run_extras_large(kda, hbm_peak, stream, extras)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rate, desc, threads, _, _ = _oracle_sample_rate(3, 12.0)
        cpu = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": kda.PREFILL_COMPUTE_DTYPE, "data": "synthetic",
            "config": {"workload": cfg.name, "T": T, "H": H, "d": D, "chunk": 64,
                       "qkv": "bf16", "gates": "f32", "state": "f32",
                       "l2": f"inputs larger than L2 ({step_bytes / 1e9:.1f} GB per step)",
                       "parallelism": f"replicas x{ws}"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak,
                         "frac_nominal_8tbs": achieved / 8000.0,
                         "tensor_pipe_pct": _profiled_metric("tensor_pipe_active_pct"),
                         "traffic": _profiled_traffic(split, T * H),
                         "traffic_note": ("DRAM bytes of one call from the one-pass ncu capture "
                                          "of the same call, profiles/kda_chunk_tc_longctx_dram.md;"
                                          " null if the kernel changed since"),
                         "peak_kind": peak_kind,
                         "kernel": "kda_chunk_tc_kernel",
                         "unit_of_work": (f"one prefill call split in {n_seg} segments "
                                          "(zero-state pass + segment scan + correction pass)"
                                          if split else "one launch"),
                         "algorithmic_bytes_per_call": step_bytes,
                         "avg_call_ms": avg_launch_ms},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps * launches_per_call,
            "clocks": clocks,
            "decode": {"workload": dcfg.name, "steps": args.decode_steps,
                       "us_per_step": dec_step_us, "GBps": dec_gbs,
                       "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": hbm_peak,
                                    "unit": "GB/s", "frac": dec_gbs / (hbm_peak * ws),
                                    "algorithmic_bytes_per_step": chains * DECODE_BYTES_PER_CHAIN},
                       "gpu_launches": args.decode_steps,
                       "l2": "state 512 MiB > L2"},
            "extras": extras if extras is not None else "skipped (N > 1 or --no-extras)",
            "decode_tokens": {"workload": f"{dcfg.name}_t{t_dec}", "calls": dt_calls,
                              "tokens_per_call": t_dec,
                              "us_per_call": dt_ms / dt_calls * 1e3,
                              "tokens_per_s": dt_tok_s, "GBps": dt_gbs,
                              "roofline": {"bound": "hbm", "achieved": dt_gbs, "peak": hbm_peak,
                                           "unit": "GB/s", "frac": dt_gbs / (hbm_peak * ws),
                                           "algorithmic_bytes_per_call": dt_bytes},
                              "gpu_launches": dt_calls,
                              "l2": "state 512 MiB > L2"},
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

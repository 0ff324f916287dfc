"""GPU parity: the CUDA kernels (through the C ABI) against the fp64 oracle.

Error metric (global, as the tolerance is stated): max|x - x_ref| / max|x_ref|
over the whole compared tensor. Bounds: 1e-4 for fp32 inputs, 2e-2 for bf16
inputs with an fp32 state, for both o and the final state.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import kda_inputs
import oracle

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def rel_err(x, ref):
    x = x.detach().double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)
    ref = np.asarray(ref)
    den = np.abs(ref).max()
    return float(np.abs(x - ref).max() / (den if den > 0 else 1.0))


@pytest.fixture(scope="module")
def kda():
    from channel_wise_gated_b200 import build
    build.build()
    import channel_wise_gated_b200 as m
    return m


@pytest.fixture(autouse=True)
def _no_device_error(request, kda):
    """Every launch must finish without a device-side error (a timed-out wait or a
    clamped cu_seqlens); the one test that provokes an error reads the word itself."""
    yield
    if "bad_seqlens" not in request.node.name:
        assert kda.device_status() == 0


def _oracle(inp, heads=None):
    sel = (lambda t: t[:, heads]) if heads is not None else (lambda t: t)
    h0 = inp["h0"]
    if h0 is not None and heads is not None:
        h0 = h0[:, heads]
    return oracle.oracle_forward(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]),
                                 sel(inp["log_alpha"]), sel(inp["beta"]), h0=h0,
                                 cu_seqlens=inp["cu_seqlens"].cpu(), col_block=16)


def _run(kda, inp, kernel="auto"):
    # a single sequence goes in without cu_seqlens, as bench.py passes it (this is
    # what lets a long one be split in time)
    cu = None if len(inp["lens"]) == 1 else inp["cu_seqlens"]
    return kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                         h0=inp["h0"], cu_seqlens=cu, kernel=kernel)


def _split_segments(kda, T, H):
    """Segments the time split uses for one bf16 sequence on this device (0: no split)."""
    return max(len(kda.split_plan(H, T)) - 1, 0)


@pytest.mark.parametrize("kernel", ["auto", "simt"])
def test_config0_tiny_fp32(kda, kernel):
    inp = kda_inputs.make_config(0, device="cuda")
    o, hT = _run(kda, inp, kernel)
    o_ref, h_ref = _oracle(inp)
    assert rel_err(o, o_ref) <= TOL_F32
    assert rel_err(hT, h_ref) <= TOL_F32
    assert kda.device_status() == 0


@pytest.mark.parametrize("kernel", ["auto", "simt"])
def test_config1_prefill_bf16(kda, kernel):
    inp = kda_inputs.make_config(1, device="cuda")
    o, hT = _run(kda, inp, kernel)
    o_ref, h_ref = _oracle(inp)
    e_o, e_s = rel_err(o, o_ref), rel_err(hT, h_ref)
    print(f"config1 {kernel}: o {e_o:.2e} hT {e_s:.2e}")
    assert e_o <= TOL_BF16 and e_s <= TOL_BF16


def test_config2_varlen(kda):
    inp = kda_inputs.make_config(2, device="cuda")
    assert len(inp["lens"]) == 16
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)   # all 32 heads, every sequence, every token
    e_o = rel_err(o, o_ref)
    e_s = rel_err(hT, h_ref)
    print(f"config2: o {e_o:.2e} hT {e_s:.2e}")
    assert e_o <= TOL_BF16 and e_s <= TOL_BF16
    assert kda.device_status() == 0


def test_config3_long_context(kda):
    """Full 1,048,576-token launch; the oracle follows 2 sampled heads end to end."""
    inp = kda_inputs.make_config(3, device="cuda")
    o, hT = _run(kda, inp)
    heads = [5, 26]
    o_ref, h_ref = _oracle(inp, heads)
    e_o = rel_err(o[:, heads], o_ref)
    e_s = rel_err(hT[:, heads], h_ref)
    print(f"config3: o {e_o:.2e} hT {e_s:.2e}")
    assert e_o <= TOL_BF16 and e_s <= TOL_BF16
    # the tail of the sequence separately (errors must not grow along the sequence)
    assert rel_err(o[-4096:, heads], o_ref[-4096:]) <= TOL_BF16
    del inp, o, hT
    torch.cuda.empty_cache()


def test_config4_decode(kda):
    """1000 in-place decode steps for all 8,192 states; oracle on 64 sampled chains."""
    c = kda_inputs.DECODE_CONFIG
    inp = kda_inputs.make_decode_config(device="cuda")
    state = inp["state"].clone()
    outs = []
    for s in range(c.steps):
        outs.append(kda.decode_step(inp["q"][s], inp["k"][s], inp["v"][s],
                                    inp["log_alpha"][s], inp["beta"][s], state))
    o = torch.stack(outs)
    g = torch.Generator().manual_seed(44)
    flat = torch.randperm(c.n_seqs * c.n_heads, generator=g)[:64]
    seqs, heads = (flat // c.n_heads).tolist(), (flat % c.n_heads).tolist()
    pick = lambda t: torch.stack([t[:, n, h] for n, h in zip(seqs, heads)], dim=1)[:, :, None]
    st0 = torch.stack([inp["state"][n, h] for n, h in zip(seqs, heads)])[:, None]
    o_ref, s_ref = oracle.oracle_decode_steps(pick(inp["q"]), pick(inp["k"]), pick(inp["v"]),
                                              pick(inp["log_alpha"]), pick(inp["beta"]), st0,
                                              col_block=32)
    o_gpu = torch.stack([o[:, n, h] for n, h in zip(seqs, heads)], dim=1)[:, :, None]
    s_gpu = torch.stack([state[n, h] for n, h in zip(seqs, heads)])[:, None]
    e_o, e_s = rel_err(o_gpu, o_ref), rel_err(s_gpu, s_ref)
    print(f"config4: o {e_o:.2e} state {e_s:.2e}")
    assert e_o <= TOL_BF16 and e_s <= TOL_BF16


def test_decode_fp32_exact(kda):
    inp = kda_inputs.make_decode(3, 4, 20, torch.float32, torch.float32, seed=9, device="cuda")
    state = inp["state"].clone()
    o = torch.stack([kda.decode_step(inp["q"][s], inp["k"][s], inp["v"][s], inp["log_alpha"][s],
                                     inp["beta"][s], state) for s in range(20)])
    o_ref, s_ref = oracle.oracle_decode_steps(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                              inp["beta"], inp["state"])
    assert rel_err(o, o_ref) <= TOL_F32
    assert rel_err(state, s_ref) <= TOL_F32


@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 200])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_ragged_lengths(kda, T, dtype):
    inp = kda_inputs.make_prefill([T], 3, dtype, torch.float32, 3.0, True, seed=T, device="cuda")
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert rel_err(o, o_ref) <= tol
    assert rel_err(hT, h_ref) <= tol


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_varlen_with_empty_and_tiny_sequences(kda, dtype):
    lens = [0, 1, 130, 0, 64, 7]
    inp = kda_inputs.make_prefill(lens, 2, dtype, torch.float32, 3.0, True, seed=21, device="cuda")
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert rel_err(o, o_ref) <= tol
    assert rel_err(hT, h_ref) <= tol
    # an empty sequence returns its initial state unchanged
    assert torch.equal(hT[0], inp["h0"][0]) and torch.equal(hT[3], inp["h0"][3])
    assert kda.device_status() == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_strong_decay_stress(kda, dtype):
    """log alpha around -5 per token: chunk decay spans hundreds of nats."""
    inp = kda_inputs.make_prefill([300], 2, dtype, torch.float32, -5.0, True, seed=31,
                                  device="cuda")
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert rel_err(o, o_ref) <= tol
    assert rel_err(hT, h_ref) <= max(tol, 1e-30)


def test_time_split_32_heads_ragged(kda):
    """One long sequence split in time (3 segments at 32 heads), random h0, ragged tail."""
    T, H = 64 * 60 + 37, 32
    assert _split_segments(kda, T, H) == 3
    inp = kda_inputs.make_prefill([T], H, torch.bfloat16, torch.float32, 3.0, True, seed=81,
                                  device="cuda")
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)
    assert rel_err(o, o_ref) <= TOL_BF16
    assert rel_err(hT, h_ref) <= TOL_BF16


def test_time_split_16_heads_mixed_decay(kda):
    """16 heads split into 5 segments; strong-decay chunks put exact-path chunks into
    every pass (the transition runs start from the identity with v = 0, the
    corrections from the segments' entering states)."""
    T, H = 64 * 100 + 5, 16
    assert _split_segments(kda, T, H) == 5
    inp = kda_inputs.make_prefill([T], H, torch.bfloat16, torch.float32, 3.0, True, seed=82,
                                  device="cuda")
    g = torch.Generator(device="cuda").manual_seed(83)
    la = inp["log_alpha"]
    for c in (3, 17, 18, 40, 41, 70, 99):
        rows = slice(64 * c, 64 * c + 64)
        x = torch.randn(la[rows].shape, generator=g, device="cuda") - 5.0
        la[rows] = torch.nn.functional.logsigmoid(x)
    # and slow decay elsewhere, so that segment transitions do not vanish
    slow = torch.ones(T, dtype=torch.bool, device="cuda")
    for c in (3, 17, 18, 40, 41, 70, 99):
        slow[64 * c:64 * c + 64] = False
    la[slow] *= 0.05
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)
    assert rel_err(o, o_ref) <= TOL_BF16
    assert rel_err(hT, h_ref) <= TOL_BF16


def test_packed_batch_longest_first(kda):
    """A packed batch with more CTAs than SMs is launched longest sequence first (the
    order lives in the workspace): same results as index order, and the oracle's."""
    lens = [64 * 3 + 5, 0, 900, 64, 1, 2000, 64 * 20, 333, 0, 1500] * 4
    H = 16
    assert len(lens) * H > 148
    inp = kda_inputs.make_prefill(lens, H, torch.bfloat16, torch.float32, 3.0, True, seed=85,
                                  device="cuda")
    lib = kda._native.load()
    assert lib.kda_chunk_fwd_workspace_size(len(lens), sum(lens), H, kda._native.KDA_BF16, 1) > 0
    o_a, h_a = _run(kda, inp, kernel="auto")      # ordered (workspace)
    o_s, h_s = _run(kda, inp, kernel="single")    # index order (no workspace)
    assert torch.equal(o_a, o_s) and torch.equal(h_a, h_s)
    o_ref, h_ref = _oracle(inp)
    assert rel_err(o_a, o_ref) <= TOL_BF16
    assert rel_err(h_a, h_ref) <= TOL_BF16


def test_time_split_equals_single_pass(kda):
    """The split and the single pass compute the same recurrence."""
    T, H = 64 * 64, 32
    inp = kda_inputs.make_prefill([T], H, torch.bfloat16, torch.float32, 3.0, True, seed=84,
                                  device="cuda")
    o_s, h_s = _run(kda, inp, kernel="auto")
    o_1, h_1 = _run(kda, inp, kernel="single")
    assert _split_segments(kda, T, H) == 3
    assert rel_err(o_s, o_1.double().cpu().numpy()) <= TOL_BF16
    assert rel_err(h_s, h_1.double().cpu().numpy()) <= TOL_BF16


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_mixed_decay_regimes(kda, dtype):
    """Chunks of ordinary decay interleaved with chunks of very strong decay (whose
    within-chunk range exceeds any fixed factorisation) and chunks whose range sits
    right at the 60-nat boundary, some channels on either side of it."""
    T, H = 704, 2
    inp = kda_inputs.make_prefill([T], H, dtype, torch.float32, 3.0, True, seed=33,
                                  device="cuda")
    g = torch.Generator(device="cuda").manual_seed(34)
    la = inp["log_alpha"]
    for c, mu in ((1, -5.0), (2, -5.0), (4, -0.45), (5, -5.0), (7, -0.45), (8, -0.45), (10, -5.0)):
        rows = slice(64 * c, min(T, 64 * c + 64))
        x = torch.randn(la[rows].shape, generator=g, device="cuda") + mu
        la[rows] = torch.nn.functional.logsigmoid(x)
    o, hT = _run(kda, inp)
    assert kda.device_status() == 0
    o_ref, h_ref = _oracle(inp)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert rel_err(o, o_ref) <= tol
    assert rel_err(hT, h_ref) <= tol


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_no_decay_full_erase(kda, dtype):
    """alpha = 1 (log alpha = 0) and beta = 1: pure DeltaNet with full erase strength."""
    inp = kda_inputs.make_prefill([192], 2, dtype, torch.float32, 3.0, False, seed=41,
                                  device="cuda")
    inp["log_alpha"].zero_()
    inp["beta"].fill_(1.0)
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert rel_err(o, o_ref) <= tol
    assert rel_err(hT, h_ref) <= tol


def test_zero_tokens_and_optional_outputs(kda):
    inp = kda_inputs.make_prefill([0], 2, torch.bfloat16, torch.float32, 3.0, True, seed=1,
                                  device="cuda")
    o, hT = _run(kda, inp)
    assert o.shape[0] == 0 and torch.equal(hT, inp["h0"])
    inp = kda_inputs.make_prefill([100], 2, torch.bfloat16, torch.float32, 3.0, False, seed=2,
                                  device="cuda")
    o1, _ = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                          output_final_state=False)
    o2, _ = _run(kda, inp)
    assert torch.equal(o1, o2)


def test_chunk_equals_decode_iterated(kda):
    """Chunkwise prefill and the recurrent step agree on the same inputs."""
    N, H, T = 2, 4, 150
    inp = kda_inputs.make_prefill([T] * N, H, torch.bfloat16, torch.float32, 3.0, True, seed=51,
                                  device="cuda")
    o_chunk, h_chunk = _run(kda, inp)
    state = inp["h0"].clone()
    o_dec = torch.empty_like(o_chunk)
    for t in range(T):
        idx = torch.tensor([t, T + t], device="cuda")
        o_dec[idx] = kda.decode_step(inp["q"][idx], inp["k"][idx], inp["v"][idx],
                                     inp["log_alpha"][idx].contiguous(),
                                     inp["beta"][idx].contiguous(), state)
    o_ref, h_ref = _oracle(inp)
    assert rel_err(o_chunk, o_dec.double().cpu().numpy()) <= TOL_BF16
    assert rel_err(h_chunk, state.double().cpu().numpy()) <= TOL_BF16
    assert rel_err(o_dec, o_ref) <= TOL_BF16


def test_prefill_then_decode_resumes(kda):
    """Checkpoint/resume: prefill(T) then one decode step equals prefill(T+1)."""
    T, H = 129, 3
    inp = kda_inputs.make_prefill([T + 1], H, torch.float32, torch.float32, 3.0, True, seed=61,
                                  device="cuda")
    sl = lambda t, a, b: t[a:b].contiguous()
    _, hT = kda.chunk_fwd(sl(inp["q"], 0, T), sl(inp["k"], 0, T), sl(inp["v"], 0, T),
                          sl(inp["log_alpha"], 0, T), sl(inp["beta"], 0, T), h0=inp["h0"])
    state = hT[0:1].clone()
    o_last = kda.decode_step(sl(inp["q"], T, T + 1), sl(inp["k"], T, T + 1),
                             sl(inp["v"], T, T + 1), sl(inp["log_alpha"], T, T + 1),
                             sl(inp["beta"], T, T + 1), state)
    o_full, h_full = _run(kda, inp)
    assert rel_err(o_last, o_full[T:T + 1].double().cpu().numpy()) <= TOL_F32
    assert rel_err(state, h_full.double().cpu().numpy()) <= TOL_F32


def test_bad_seqlens_are_clamped_and_reported(kda):
    inp = kda_inputs.make_prefill([100, 100], 2, torch.bfloat16, torch.float32, 3.0, False,
                                  seed=71, device="cuda")
    cu = torch.tensor([0, 150, 120], dtype=torch.int32, device="cuda")   # not monotone
    kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], cu_seqlens=cu)
    assert kda.device_status() == kda._native.KDA_ERR_SEQLENS
    assert kda.device_status() == 0   # read clears it


@pytest.mark.parametrize("eps", [1e-1, 1e-2])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_nearly_parallel_keys_full_erase(kda, eps, dtype):
    """The triangular solve's hard case: runs of nearly parallel unit keys, erase
    strength beta in [0.98, 1], decay close to one and a large initial state (std 1),
    so that I + A is close to singular within a run and T = (I + A)^-1 is far from
    the identity. bf16 takes the tensor-core kernel (T beta rounded to bf16 as an
    MMA operand), fp32 the CUDA-core kernel."""
    T, H = 64 * 6 + 17, 4
    for run in (16, 64):
        inp = kda_inputs.make_parallel_keys(T, H, dtype, eps=eps, run=run,
                                            seed=int(1e4 * eps) + run, device="cuda")
        o, hT = _run(kda, inp)
        o_ref, h_ref = _oracle(inp)
        tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
        e_o, e_s = rel_err(o, o_ref), rel_err(hT, h_ref)
        print(f"parallel keys eps={eps} run={run} {dtype}: o {e_o:.2e} hT {e_s:.2e}")
        assert e_o <= tol and e_s <= tol


def test_nearly_parallel_keys_time_split(kda):
    """The same hard case through the time split (32 heads, 3 segments): the segment
    transitions barely shrink, and the state enters every segment large."""
    T, H = 64 * 60 + 9, 32
    assert _split_segments(kda, T, H) == 3
    inp = kda_inputs.make_parallel_keys(T, H, torch.bfloat16, eps=1e-2, run=32, seed=77,
                                        device="cuda")
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)
    e_o, e_s = rel_err(o, o_ref), rel_err(hT, h_ref)
    print(f"parallel keys, split: o {e_o:.2e} hT {e_s:.2e}")
    assert e_o <= TOL_BF16 and e_s <= TOL_BF16


def test_time_split_uneven_segments_4_heads(kda):
    """4 heads over 321 chunks (the last one ragged): 17 segments whose lengths differ
    by one chunk (the chunk count is not a multiple of the segment count)."""
    T, H = 320 * 64 + 13, 4
    bounds = kda.split_plan(H, T)
    assert len(bounds) - 1 == 17
    sizes = np.diff(bounds)
    assert bounds[0] == 0 and bounds[-1] == T and sizes.min() > 15 * 64   # >= 16 chunks
    assert len(set(sizes[:-1].tolist())) == 2   # 19 and 18 chunks
    inp = kda_inputs.make_prefill([T], H, torch.bfloat16, torch.float32, 3.0, True, seed=86,
                                  device="cuda")
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)
    e_o, e_s = rel_err(o, o_ref), rel_err(hT, h_ref)
    print(f"4 heads, 17 segments: o {e_o:.2e} hT {e_s:.2e}")
    assert e_o <= TOL_BF16 and e_s <= TOL_BF16
    o_1, h_1 = _run(kda, inp, kernel="single")
    assert rel_err(o, o_1.double().cpu().numpy()) <= TOL_BF16
    assert rel_err(hT, h_1.double().cpu().numpy()) <= TOL_BF16


@pytest.mark.parametrize("x_mean", [0.0, -5.0])
def test_time_split_transitions_vanish(kda, x_mean):
    """Strong decay (about -50 or -320 nats per chunk): every segment transition M_j
    and every correction becomes exactly zero after a chunk or two, so its CTA stops
    early while the other roles are still ahead of it. Results must match the oracle
    and the single pass."""
    T, H = 64 * 100 + 5, 16
    assert _split_segments(kda, T, H) == 5
    inp = kda_inputs.make_prefill([T], H, torch.bfloat16, torch.float32, x_mean, True, seed=87,
                                  device="cuda")
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)
    e_o, e_s = rel_err(o, o_ref), rel_err(hT, h_ref)
    print(f"transitions vanish (mu {x_mean}): o {e_o:.2e} hT {e_s:.2e}")
    assert e_o <= TOL_BF16 and e_s <= max(TOL_BF16, 1e-30)
    o_1, h_1 = _run(kda, inp, kernel="single")
    assert rel_err(o, o_1.double().cpu().numpy()) <= TOL_BF16


def test_time_split_two_segments(kda):
    """48 heads over 256 chunks: 2 segments (no transition chain, no scan: the correction
    starts from segment 0's final state), ragged tail, random h0."""
    T, H = 256 * 64 - 21, 48
    assert _split_segments(kda, T, H) == 2
    inp = kda_inputs.make_prefill([T], H, torch.bfloat16, torch.float32, 3.0, True, seed=89,
                                  device="cuda")
    o, hT = _run(kda, inp)
    o_ref, h_ref = _oracle(inp)
    e_o, e_s = rel_err(o, o_ref), rel_err(hT, h_ref)
    print(f"2 segments: o {e_o:.2e} hT {e_s:.2e}")
    assert e_o <= TOL_BF16 and e_s <= TOL_BF16


def test_time_split_long_segments(kda):
    """32 heads over 3000 chunks: 4 segments of 750 chunks, with the transition runs
    and the corrections expected to end early (the long-context plan at a fifth of
    its length). The oracle follows 3 heads end to end."""
    T, H = 3000 * 64, 32
    assert _split_segments(kda, T, H) == 4
    inp = kda_inputs.make_prefill([T], H, torch.bfloat16, torch.float32, 4.0, True, seed=88,
                                  device="cuda")
    o, hT = _run(kda, inp)
    heads = [0, 17, 31]
    o_ref, h_ref = _oracle(inp, heads)
    e_o, e_s = rel_err(o[:, heads], o_ref), rel_err(hT[:, heads], h_ref)
    print(f"4 segments of 750 chunks: o {e_o:.2e} hT {e_s:.2e}")
    assert e_o <= TOL_BF16 and e_s <= TOL_BF16

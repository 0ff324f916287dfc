"""The oracle against its pins (CPU only), plus a mutation test of the pins."""

from __future__ import annotations

import functools
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle.oracle_forward)


def test_column_blocks_are_bitwise_identical():
    """Splitting value columns into tasks changes no arithmetic of any column."""
    rng = np.random.default_rng(11)
    T, H, dk, dv = 50, 3, 8, 10
    q = rng.standard_normal((T, H, dk)).astype(np.float32)
    k = rng.standard_normal((T, H, dk)).astype(np.float32)
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    la = (-rng.random((T, H, dk))).astype(np.float32)
    b = rng.random((T, H)).astype(np.float32)
    o1, s1 = oracle.oracle_forward(q, k, v, la, b, col_block=0)
    o2, s2 = oracle.oracle_forward(q, k, v, la, b, col_block=3)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


def test_varlen_equals_separate_sequences():
    """Packing sequences with cu_seqlens equals running each one on its own."""
    rng = np.random.default_rng(12)
    lens = [5, 1, 17, 9]
    H, dk, dv = 2, 6, 5
    T = sum(lens)
    q = rng.standard_normal((T, H, dk)).astype(np.float32)
    k = rng.standard_normal((T, H, dk)).astype(np.float32)
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    la = (-rng.random((T, H, dk))).astype(np.float32)
    b = rng.random((T, H)).astype(np.float32)
    h0 = rng.standard_normal((len(lens), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, hT = oracle.oracle_forward(q, k, v, la, b, h0=h0, cu_seqlens=cu)
    for n, (a, e) in enumerate(zip(cu[:-1], cu[1:])):
        on, hn = oracle.oracle_forward(q[a:e], k[a:e], v[a:e], la[a:e], b[a:e], h0=h0[n:n + 1])
        np.testing.assert_array_equal(o[a:e], on)
        np.testing.assert_array_equal(hT[n], hn[0])


def test_resume_from_state():
    """Running T tokens equals running a prefix and resuming from its final state."""
    rng = np.random.default_rng(13)
    T, H, dk, dv = 30, 2, 5, 4
    q = rng.standard_normal((T, H, dk)).astype(np.float32)
    k = rng.standard_normal((T, H, dk)).astype(np.float32)
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    la = (-rng.random((T, H, dk))).astype(np.float32)
    b = rng.random((T, H)).astype(np.float32)
    o, hT = oracle.oracle_forward(q, k, v, la, b)
    o1, h1 = oracle.oracle_forward(q[:11], k[:11], v[:11], la[:11], b[:11])
    o2, h2 = oracle.oracle_forward(q[11:], k[11:], v[11:], la[11:], b[11:], h0=h1)
    np.testing.assert_allclose(np.concatenate([o1, o2]), o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(h2, hT, rtol=1e-13, atol=1e-14)


def test_decode_steps_is_the_same_recurrence():
    rng = np.random.default_rng(14)
    steps, N, H, dk, dv = 4, 3, 2, 5, 4
    q = rng.standard_normal((steps, N, H, dk)).astype(np.float32)
    k = rng.standard_normal((steps, N, H, dk)).astype(np.float32)
    v = rng.standard_normal((steps, N, H, dv)).astype(np.float32)
    la = (-rng.random((steps, N, H, dk))).astype(np.float32)
    b = rng.random((steps, N, H)).astype(np.float32)
    st = rng.standard_normal((N, H, dk, dv))
    o, s = oracle.oracle_decode_steps(q, k, v, la, b, st)
    for n in range(N):
        on, sn = oracle.oracle_forward(q[:, n], k[:, n], v[:, n], la[:, n], b[:, n],
                                       h0=st[n:n + 1])
        np.testing.assert_array_equal(o[:, n], on)
        np.testing.assert_array_equal(s[n], sn[0])


# ---------------------------------------------------------------------------
# Mutation test: plant one plausible mistake at a time into a copy of the C
# oracle, build it, and check that at least one pin rejects it.
# ---------------------------------------------------------------------------

_FORGET = ("    for (int64_t c = 0; c < dk; ++c)\n"
           "      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] *= alpha[c];\n")
_ERASE_HEAD = "    /* 2. erase:"
_WRITE_HEAD = "    /* 3. write:"
_READ_HEAD = "    /* 4. read:"

MUTANTS = {
    # beta dropped from the write term (the garbled DPLR line of the deep-dive page)
    "write_without_beta": [("S[c * nc + j] += bk * (double)vt[j0 + j];",
                            "S[c * nc + j] += (double)kt[c] * (double)vt[j0 + j];")],
    # sign error in the erase
    "erase_sign": [("S[c * nc + j] -= bk * u[j];", "S[c * nc + j] += bk * u[j];")],
    # erase projects with q instead of k
    "erase_with_q": [("const double kc = (double)kt[c];", "const double kc = (double)qt[c];")],
    # log-decay used as if it were the decay itself
    "no_exp_on_gate": [("alpha[c] = exp((double)lat[c]);", "alpha[c] = 1.0 + (double)lat[c];")],
    # decay applied along the value axis instead of the key axis
    "decay_wrong_axis": [("S[c * nc + j] *= alpha[c];", "S[c * nc + j] *= alpha[(j0 + j) % dk];")],
    # decay applied after the delta correction (GDN order; wrong once alpha varies by channel)
    "decay_after_erase": [(_FORGET, ""), (_WRITE_HEAD, _FORGET + _WRITE_HEAD)],
    # decay applied after the write
    "decay_last": [(_FORGET, ""), (_READ_HEAD, _FORGET + _READ_HEAD)],
    # output read from the state before the update (exclusive instead of inclusive)
    "read_before_update": [
        ("    /* 1. forget: S <- Diag(alpha_t) S */\n",
         "    { double* ot0 = o + (t * n_heads + h) * dv;\n"
         "      for (int64_t j = 0; j < nc; ++j) { double a = 0.0;\n"
         "        for (int64_t c = 0; c < dk; ++c) a += (double)qt[c] * S[c * nc + j];\n"
         "        ot0[j0 + j] = a; } }\n"
         "    /* 1. forget: S <- Diag(alpha_t) S */\n"),
        ("    for (int64_t j = 0; j < nc; ++j) ot[j0 + j] = u[j];\n", "")],
    # initial state read transposed
    "h0_transposed": [("S[c * nc + j] = h0 ? h0[c * dv + j0 + j] : 0.0;",
                       "S[c * nc + j] = h0 ? h0[(j0 + j) * dk + c] : 0.0;")],
    # the read uses a decayed copy once more
    "double_decay_on_read": [("u[j] += qc * S[c * nc + j];", "u[j] += qc * S[c * nc + j] * alpha[c];")],
}


# Mistakes planted into the Gated DeltaNet chain (the scalar gate commutes with the
# erase, so the order of those two is not a mistake; the others are).
_GATE = ("    for (int64_t c = 0; c < dk; ++c)\n"
         "      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] *= at;\n")
GDN_MUTANTS = {
    "gdn_no_exp_on_gate": [("const double at = exp((double)log_a[t * n_heads + h]);",
                            "const double at = 1.0 + (double)log_a[t * n_heads + h];")],
    "gdn_gate_dropped": [(_GATE, "")],
    "gdn_gate_after_write": [(_GATE, ""), ("    /* 4. read: o_t = S^T q_t */\n",
                                           _GATE + "    /* 4. read: o_t = S^T q_t */\n")],
    "gdn_gate_of_next_token": [("exp((double)log_a[t * n_heads + h])",
                                "exp((double)log_a[(t + 1 < eos ? t + 1 : t) * n_heads + h])")],
    "gdn_erase_sign": [("S[c * nc + j] -= bk * u[j];", "S[c * nc + j] += bk * u[j];")],
}

_GDN_MARK = "static int run_gdn_chain("
_DPLR_MARK = "static int run_dplr_chain("

# Mistakes planted into the DPLR chain.
DPLR_MUTANTS = {
    "dplr_ab_swapped": [("const double bc = (double)bt[c];", "const double bc = (double)at[c];"),
                        ("const double ac = (double)at[c];", "const double ac = (double)bt[c];")],
    "dplr_read_after_forget": [
        ("    /* 1. low-rank read of the old state: u = b^T S */\n",
         "    for (int64_t c = 0; c < dk; ++c) { const double al0 = exp((double)lat[c]);\n"
         "      for (int64_t j = 0; j < nc; ++j) S[c * nc + j] *= al0; }\n"),
        ("    /* 2. forget: S <- Diag(alpha) S */\n    for (int64_t c = 0; c < dk; ++c) {\n"
         "      const double al = exp((double)lat[c]);\n",
         "    for (int64_t c = 0; c < dk; ++c) {\n      const double al = 1.0;\n")],
    "dplr_correction_sign": [("S[c * nc + j] -= ac * u[j];", "S[c * nc + j] += ac * u[j];")],
    "dplr_no_forget": [("      const double al = exp((double)lat[c]);", "      const double al = 1.0;")],
}


@functools.lru_cache(maxsize=None)
def _mutant_lib(name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")).read()
    # KDA mistakes go into the KDA chain only, Gated DeltaNet ones into its chain only
    c1, c2 = src.index(_GDN_MARK), src.index(_DPLR_MARK)
    parts = [src[:c1], src[c1:c2], src[c2:]]   # KDA chain, Gated DeltaNet chain, DPLR chain
    which = 1 if name in GDN_MUTANTS else (2 if name in DPLR_MUTANTS else 0)
    table = (MUTANTS, GDN_MUTANTS, DPLR_MUTANTS)[which]
    part = parts[which]
    for old, new in table[name]:
        assert part.count(old) == 1, f"mutation anchor not unique/present for {name}: {old!r}"
        part = part.replace(old, new)
    parts[which] = part
    src = "".join(parts)
    d = tempfile.mkdtemp(prefix=f"kda_mut_{name}_")
    c = os.path.join(d, "m.c")
    so = os.path.join(d, "m.so")
    with open(c, "w") as fh:
        fh.write(src)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", c, "-o", so, "-lm"],
                   check=True)
    lib = oracle.load_library(so)
    lib._tmpdir = d
    return lib


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_planted_mistake_fails_a_pin(name):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    lib = _mutant_lib(name)
    fwd = functools.partial(oracle.oracle_forward, lib=lib)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(fwd)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"


@pytest.mark.parametrize("pin", pins.ALL_GDN_PINS, ids=lambda p: p.__name__)
def test_gdn_oracle_pin(pin):
    pin(oracle.oracle_gdn_forward)


def test_gdn_equals_kda_with_a_shared_gate():
    """A scalar gate is KDA's channel-wise gate with every channel equal (the scalar
    commutes with the erase): the two oracles agree on a 128-dimensional head."""
    rng = np.random.default_rng(26)
    T, H, d = 40, 2, 128
    f = lambda a: np.asarray(a, dtype=np.float32)
    q = rng.standard_normal((T, H, d))
    k = rng.standard_normal((T, H, d))
    q, k = f(q / np.linalg.norm(q, axis=2, keepdims=True)), f(k / np.linalg.norm(k, axis=2, keepdims=True))
    v = f(rng.standard_normal((T, H, d)))
    beta = f(1.0 / (1.0 + np.exp(-rng.standard_normal((T, H)))))
    log_a = f(-rng.random((T, H)) * 0.3)
    h0 = 0.02 * rng.standard_normal((1, H, d, d))
    o_g, h_g = oracle.oracle_gdn_forward(q, k, v, log_a, beta, h0=h0)
    o_k, h_k = oracle.oracle_forward(q, k, v, np.repeat(log_a[:, :, None], d, axis=2), beta, h0=h0)
    np.testing.assert_allclose(o_g, o_k, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(h_g, h_k, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("name", sorted(GDN_MUTANTS))
def test_each_planted_gdn_mistake_fails_a_pin(name):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    lib = _mutant_lib(name)
    gfwd = functools.partial(oracle.oracle_gdn_forward, lib=lib)
    failed = []
    for pin in pins.ALL_GDN_PINS:
        try:
            pin(gfwd)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every Gated DeltaNet pin"


@pytest.mark.parametrize("pin", pins.ALL_DPLR_PINS, ids=lambda p: p.__name__)
def test_dplr_oracle_pin(pin):
    pin(oracle.oracle_dplr_forward)


@pytest.mark.parametrize("name", sorted(DPLR_MUTANTS))
def test_each_planted_dplr_mistake_fails_a_pin(name):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    lib = _mutant_lib(name)
    dfwd = functools.partial(oracle.oracle_dplr_forward, lib=lib)
    failed = []
    for pin in pins.ALL_DPLR_PINS:
        try:
            pin(dfwd)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every DPLR pin"

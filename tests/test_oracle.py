"""Pins for the fp64 oracle, against what the pages and the mathematics fix.

None of these re-types the oracle's own formula: every check compares the
oracle with something independent of it — a hand-derived worked example, the
term-by-term definition on tiny inputs, a closed form, a library routine
(numpy cumsum, torch group_norm / silu), or an invariant the pages state
(the three forms give the same value; the state summarises the past).  The
mutation tests at the end plant plausible mistakes in copies of the oracle
(on the CPU) and check that at least one pin fails for each.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, T, dk, dv):
    s = 1.0 / np.sqrt(dk)
    return (rng.standard_normal((T, dk)) * s, rng.standard_normal((T, dk)) * s,
            rng.standard_normal((T, dv)) * s)


def _rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------------------
# Pin checks, written against an implementation ``impl`` with the oracle's
# per-head signatures (so that the mutation tests can reuse them).
# ---------------------------------------------------------------------------

def check_hand_example(impl):
    """Hand-derived T=3 example (tests/golden/retention_hand_t3.json)."""
    with open(os.path.join(GOLDEN, "retention_hand_t3.json")) as f:
        g = json.load(f)
    q, k, v = (np.array(g[x], dtype=np.float64) for x in ("q", "k", "v"))
    gam = g["gamma"]
    o_ref, S_ref = np.array(g["o"]), np.array(g["S_final"])
    for chunk in (1, 2, 3, 4):
        o, S = impl.retention_chunkwise(q, k, v, gam, chunk)
        np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-14)
        np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-14)
    o, S = impl.retention_recurrent(q, k, v, gam)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(impl.retention_parallel(q, k, v, gam), o_ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(impl.retention_brute(q, k, v, gam), o_ref, rtol=0, atol=1e-14)


def check_forms_agree(impl, T=37, dk=5, dv=7, seed=1):
    """brute = parallel = recurrent = chunkwise for every chunk length."""
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T, dk, dv)
    for gam in (0.0, 0.3, 0.9, 0.96875, 1.0):
        ref = impl.retention_brute(q, k, v, gam)
        assert _rel(impl.retention_parallel(q, k, v, gam), ref) < 1e-12
        o_r, S_r = impl.retention_recurrent(q, k, v, gam)
        assert _rel(o_r, ref) < 1e-12
        for chunk in (1, 2, 3, 16, T, T + 5):
            o_c, S_c = impl.retention_chunkwise(q, k, v, gam, chunk)
            assert _rel(o_c, ref) < 1e-12, (gam, chunk)
            assert _rel(S_c, S_r) < 1e-12, (gam, chunk)


def check_gamma_zero(impl, T=19, dk=4, dv=6, seed=2):
    """gamma = 0 leaves only the diagonal: o_n = (q_n . k_n) v_n."""
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T, dk, dv)
    expect = np.einsum("td,td->t", q, k)[:, None] * v
    assert _rel(impl.retention_parallel(q, k, v, 0.0), expect) < 1e-13
    assert _rel(impl.retention_recurrent(q, k, v, 0.0)[0], expect) < 1e-13
    for chunk in (1, 4, 7, T):
        assert _rel(impl.retention_chunkwise(q, k, v, 0.0, chunk)[0], expect) < 1e-13


def check_gamma_one(impl, T=23, dk=3, dv=5, seed=3):
    """gamma = 1 is causal linear attention: o_n = q_n . cumsum_m(k_m^T v_m)."""
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T, dk, dv)
    prefix = np.cumsum(k[:, :, None] * v[:, None, :], axis=0)      # [T, dk, dv]
    expect = np.einsum("td,tde->te", q, prefix)
    assert _rel(impl.retention_parallel(q, k, v, 1.0), expect) < 1e-13
    o, S = impl.retention_recurrent(q, k, v, 1.0)
    assert _rel(o, expect) < 1e-13
    assert _rel(S, prefix[-1]) < 1e-13
    for chunk in (1, 5, 8, T):
        o, S = impl.retention_chunkwise(q, k, v, 1.0, chunk)
        assert _rel(o, expect) < 1e-13
        assert _rel(S, prefix[-1]) < 1e-13


def check_constant_rows(impl, T=40):
    """q_n = q, k_m = k, v_m = v: o_n = (q.k) v (1 - gamma^(n+1)) / (1 - gamma)."""
    q1 = np.array([0.5, -1.0, 2.0])
    k1 = np.array([1.0, 0.25, 0.5])
    v1 = np.array([2.0, -3.0, 1.0, 0.5])
    q, k, v = np.tile(q1, (T, 1)), np.tile(k1, (T, 1)), np.tile(v1, (T, 1))
    for gam in (0.5, 0.9, 0.99):
        n = np.arange(T)
        geo = (1.0 - gam ** (n + 1)) / (1.0 - gam)
        expect = (q1 @ k1) * geo[:, None] * v1[None, :]
        assert _rel(impl.retention_parallel(q, k, v, gam), expect) < 1e-13
        for chunk in (1, 3, 16):
            assert _rel(impl.retention_chunkwise(q, k, v, gam, chunk)[0], expect) < 1e-13


def check_split_resume(impl, T=50, dk=4, dv=3, seed=4):
    """The state summarises the past: splitting at t and resuming is the full run."""
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T, dk, dv)
    gam = 0.93
    o_full, S_full = impl.retention_chunkwise(q, k, v, gam, 8)
    for t in (1, 7, 8, 25, 49):
        o1, S1 = impl.retention_chunkwise(q[:t], k[:t], v[:t], gam, 8)
        o2, S2 = impl.retention_chunkwise(q[t:], k[t:], v[t:], gam, 8, S1)
        assert _rel(np.concatenate([o1, o2]), o_full) < 1e-12
        assert _rel(S2, S_full) < 1e-12


def check_linearity(impl, T=21, dk=4, dv=5, seed=5):
    """Retention is linear in each of q, k and v separately."""
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T, dk, dv)
    q2, k2, v2 = _rand(rng, T, dk, dv)
    gam = 0.8
    f = lambda a, b, c: impl.retention_chunkwise(a, b, c, gam, 6)[0]
    base = f(q, k, v)
    assert _rel(f(q + q2, k, v), base + f(q2, k, v)) < 1e-12
    assert _rel(f(q, k + k2, v), base + f(q, k2, v)) < 1e-12
    assert _rel(f(q, k, 2.5 * v + v2), 2.5 * base + f(q, k, v2)) < 1e-12
    assert _rel(f(-3.0 * q, k, v), -3.0 * base) < 1e-12


def check_decode_continuation(impl, T=30, steps=6, dk=4, dv=5, seed=6):
    """Prefill T tokens chunkwise, then single steps == chunkwise over T+steps."""
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T + steps, dk, dv)
    gam = 0.95
    o_all, S_all = impl.retention_chunkwise(q, k, v, gam, 7)
    _, S = impl.retention_chunkwise(q[:T], k[:T], v[:T], gam, 7)
    for n in range(T, T + steps):
        o_n, S = impl.recurrent_step(q[n], k[n], v[n], gam, S)
        assert _rel(o_n, o_all[n]) < 1e-12
    assert _rel(S, S_all) < 1e-12


def check_groupnorm(impl):
    """Hand example (tests/golden/groupnorm_hand.json) + torch library routines."""
    with open(os.path.join(GOLDEN, "groupnorm_hand.json")) as f:
        g = json.load(f)
    o = np.array(g["o"], dtype=np.float64)[None]          # [1 token, 2 heads, 4]
    eps = g["eps"]
    gn = impl.group_norm_heads(o, eps)
    np.testing.assert_allclose(gn[0, 0] * np.sqrt(5.0 + eps),
                               g["gn_expected_head0_times_sqrt5eps"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(gn[0, 1], g["gn_expected_head1"], atol=1e-13)
    # torch.nn.functional.group_norm with one group per head, in float64
    rng = np.random.default_rng(7)
    Ntok, H, dv = 9, 3, 8
    o = rng.standard_normal((Ntok, H, dv)) * 3.0 + 1.5
    gate = rng.standard_normal((Ntok, H, dv)) * 2.0
    w = rng.standard_normal((H, dv))
    b = rng.standard_normal((H, dv))
    ot = torch.from_numpy(o.reshape(Ntok, H * dv))
    ref_gn = torch.nn.functional.group_norm(ot, H, torch.from_numpy(w.reshape(-1)),
                                            torch.from_numpy(b.reshape(-1)), eps=1e-5)
    ref = ref_gn * torch.nn.functional.silu(torch.from_numpy(gate.reshape(Ntok, H * dv)))
    got = impl.norm_gate(o, gate, 1e-5, w, b)
    assert _rel(got.reshape(Ntok, H * dv), ref.numpy()) < 1e-13
    # invariants: mean 0 and variance sigma^2/(sigma^2+eps) before the gate; g=0 -> y=0
    gn = impl.group_norm_heads(o, 1e-5)
    assert np.abs(gn.mean(axis=-1)).max() < 1e-13
    var = o.var(axis=-1)
    np.testing.assert_allclose(gn.var(axis=-1), var / (var + 1e-5), rtol=1e-12)
    assert np.abs(impl.norm_gate(o, np.zeros_like(o))).max() == 0.0


def check_swish(impl):
    """swish(0) = 0, swish(x) - swish(-x) = x, and torch silu agreement."""
    x = np.linspace(-30, 30, 601)
    assert impl.swish(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(impl.swish(x) - impl.swish(-x), x, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(impl.swish(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy(),
                               rtol=1e-14, atol=1e-300)


ALL_PINS = [check_hand_example, check_forms_agree, check_gamma_zero, check_gamma_one,
            check_constant_rows, check_split_resume, check_linearity,
            check_decode_continuation, check_groupnorm, check_swish]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle)


# ---------------------------------------------------------------------------
# Multi-head wrappers, varlen, decode batch
# ---------------------------------------------------------------------------

def test_multihead_wrappers_match_per_head():
    rng = np.random.default_rng(11)
    B, T, H, dk, dv = 2, 33, 3, 4, 6
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    gam = np.array([0.5, 0.9, 0.99])
    o_p = oracle.msr_parallel(q, k, v, gam)
    o_r, S_r = oracle.msr_recurrent(q, k, v, gam)
    o_c, S_c = oracle.msr_chunkwise(q, k, v, gam, 8)
    for b in range(B):
        for h in range(H):
            ref = oracle.retention_brute(q[b, :, h], k[b, :, h], v[b, :, h], gam[h])
            assert _rel(o_p[b, :, h], ref) < 1e-12
            assert _rel(o_r[b, :, h], ref) < 1e-12
            assert _rel(o_c[b, :, h], ref) < 1e-12
    assert _rel(S_c, S_r) < 1e-12


def test_varlen_equals_independent_runs():
    rng = np.random.default_rng(12)
    lens = [5, 0, 17, 1, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    Tt, H, dk, dv = int(cu[-1]), 2, 3, 4
    q = rng.standard_normal((1, Tt, H, dk))
    k = rng.standard_normal((1, Tt, H, dk))
    v = rng.standard_normal((1, Tt, H, dv))
    s0 = rng.standard_normal((len(lens), H, dk, dv))
    gam = np.array([0.7, 0.95])
    o, S = oracle.msr_chunkwise_varlen(q, k, v, gam, 4, cu, s0)
    for i, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        for h in range(H):
            if b > a:
                ref_o, ref_S = oracle.retention_recurrent(q[0, a:b, h], k[0, a:b, h],
                                                          v[0, a:b, h], gam[h], s0[i, h])
                assert _rel(o[0, a:b, h], ref_o) < 1e-12
                assert _rel(S[i, h], ref_S) < 1e-12
            else:
                np.testing.assert_array_equal(S[i, h], s0[i, h])   # empty: state passes through


def test_decode_batch_matches_single():
    rng = np.random.default_rng(13)
    N, H, dk, dv = 3, 2, 4, 5
    q = rng.standard_normal((N, H, dk))
    k = rng.standard_normal((N, H, dk))
    v = rng.standard_normal((N, H, dv))
    S = rng.standard_normal((N, H, dk, dv))
    gam = np.array([0.5, 0.99])
    o, S2 = oracle.msr_recurrent_step(q, k, v, gam, S)
    for n in range(N):
        for h in range(H):
            # update-then-read written out with explicit loops over the matrix entries
            Sn = np.empty((dk, dv))
            for i in range(dk):
                for j in range(dv):
                    Sn[i, j] = gam[h] * S[n, h, i, j] + k[n, h, i] * v[n, h, j]
            on = np.array([sum(q[n, h, i] * Sn[i, j] for i in range(dk)) for j in range(dv)])
            assert _rel(S2[n, h], Sn) < 1e-14
            assert _rel(o[n, h], on) < 1e-14


# ---------------------------------------------------------------------------
# Mutation tests: a plausible mistake in the oracle must fail some pin.
# ---------------------------------------------------------------------------

class _Mutant:
    """A copy of the oracle's per-head API with one function replaced."""

    def __init__(self, **over):
        for name in ("retention_brute", "retention_parallel", "retention_recurrent",
                     "retention_chunkwise", "recurrent_step", "group_norm_heads",
                     "swish", "norm_gate"):
            setattr(self, name, over.get(name, getattr(oracle, name)))


def _chunkwise_variant(read_pow_offset=1, zeta_rev=False, state_transposed=False,
                       decay_whole_chunk=True):
    def f(q, k, v, gamma, chunk, state=None):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        T, dk, dv = q.shape[0], q.shape[1], v.shape[1]
        S = np.zeros((dk, dv)) if state is None else np.array(state, dtype=np.float64)
        o = np.zeros((T, dv))
        for s in range(0, T, chunk):
            L = min(chunk, T - s)
            Qc, Kc, Vc = q[s:s + L], k[s:s + L], v[s:s + L]
            inner = ((Qc @ Kc.T) * oracle.decay_mask(gamma, L)) @ Vc
            rs = np.power(gamma, np.arange(read_pow_offset, L + read_pow_offset))
            o[s:s + L] = inner + rs[:, None] * (Qc @ S)
            ex = np.arange(L) if zeta_rev else np.arange(L - 1, -1, -1)
            upd = Kc.T @ (np.power(gamma, ex)[:, None] * Vc)
            if state_transposed and dk == dv:
                upd = upd.T
            S = (gamma ** (L if decay_whole_chunk else L - 1)) * S + upd
        return o, S
    return f


def _fails(pins, impl):
    failed = []
    for pin in pins:
        try:
            pin(impl)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    return failed


MUTANTS = {
    "chunk read decays by gamma^i instead of gamma^(i+1)":
        _Mutant(retention_chunkwise=_chunkwise_variant(read_pow_offset=0)),
    "chunk state weights reversed (gamma^j instead of gamma^(L-1-j))":
        _Mutant(retention_chunkwise=_chunkwise_variant(zeta_rev=True)),
    "state decays by gamma^(L-1) per chunk":
        _Mutant(retention_chunkwise=_chunkwise_variant(decay_whole_chunk=False)),
    "parallel mask without the diagonal":
        _Mutant(retention_parallel=lambda q, k, v, g: ((np.asarray(q) @ np.asarray(k).T)
                                                       * np.tril(oracle.decay_mask(g, len(q)), -1))
                @ np.asarray(v)),
    "parallel mask anti-causal (gamma^(m-n))":
        _Mutant(retention_parallel=lambda q, k, v, g: ((np.asarray(q) @ np.asarray(k).T)
                                                       * oracle.decay_mask(g, len(q)).T)
                @ np.asarray(v)),
    "recurrent reads before it updates":
        _Mutant(recurrent_step=lambda qn, kn, vn, g, S: (np.asarray(qn) @ np.asarray(S),
                                                          g * np.asarray(S) + np.outer(kn, vn))),
    "recurrent state v^T k (transposed operand)":
        _Mutant(recurrent_step=lambda qn, kn, vn, g, S: (
            np.asarray(qn) @ (g * np.asarray(S) + np.outer(vn, kn)[:len(qn), :np.asarray(S).shape[1]]),
            g * np.asarray(S) + np.outer(vn, kn)[:len(qn), :np.asarray(S).shape[1]])),
    "GroupNorm with unbiased variance":
        _Mutant(group_norm_heads=lambda o, eps=1e-5, weight=None, bias=None:
                (np.asarray(o) - np.asarray(o).mean(-1, keepdims=True))
                / np.sqrt(np.asarray(o).var(-1, ddof=1, keepdims=True) + eps)),
    "swish as sigmoid only":
        _Mutant(swish=lambda x: 1.0 / (1.0 + np.exp(-np.asarray(x, dtype=np.float64)))),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_pins_catch_mutant(name):
    mut = MUTANTS[name]
    # the mutant's recurrent_step must also drive its recurrent form
    if mut.recurrent_step is not oracle.recurrent_step:
        step = mut.recurrent_step

        def rec(q, k, v, gamma, state=None):
            q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
            S = np.zeros((q.shape[1], v.shape[1])) if state is None else np.asarray(state)
            o = np.zeros((q.shape[0], v.shape[1]))
            for n in range(q.shape[0]):
                o[n], S = step(q[n], k[n], v[n], gamma, S)
            return o, S
        mut.retention_recurrent = rec
    if mut.group_norm_heads is not oracle.group_norm_heads or mut.swish is not oracle.swish:
        gn, sw = mut.group_norm_heads, mut.swish
        mut.norm_gate = lambda o, g, eps=1e-5, weight=None, bias=None: (
            (gn(o, eps) * (1.0 if weight is None else np.asarray(weight))
             + (0.0 if bias is None else np.asarray(bias))) * sw(np.asarray(g).reshape(np.shape(o))))
    failed = _fails(ALL_PINS, mut)
    assert failed, f"no pin catches the mutant: {name}"

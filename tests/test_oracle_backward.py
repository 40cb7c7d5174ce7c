"""Pins for the oracle's backward (gradients of the definition).

None of these re-types the gradient formulas.  The main pin differentiates
the forward numerically: the loss L = <dO, o> + <dS_T, S_T>, evaluated with
the oracle's *recurrent* form (an independent route through the definition),
is affine in every single input entry, so a central difference over any step
gives that entry's partial derivative exactly up to rounding.  Closed forms
at gamma = 0 and gamma = 1 (cumulative sums of outer products) and the
independence of packed sequences pin the rest.  The mutation tests plant
plausible mistakes in copies of the backward, on the CPU, and check that the
finite-difference pin catches each.
"""

import numpy as np
import pytest

import oracle


def _inputs(rng, T, dk, dv, with_state=True):
    s = 1.0 / np.sqrt(dk)
    q = rng.standard_normal((T, dk)) * s
    k = rng.standard_normal((T, dk)) * s
    v = rng.standard_normal((T, dv)) * s
    do = rng.standard_normal((T, dv))
    S0 = rng.standard_normal((dk, dv)) if with_state else None
    dS = rng.standard_normal((dk, dv)) if with_state else None
    return q, k, v, do, S0, dS


def _loss(q, k, v, gamma, do, S0, dS):
    o, S = oracle.retention_recurrent(q, k, v, gamma, S0)
    L = float(np.sum(do * o))
    if dS is not None:
        L += float(np.sum(dS * S))
    return L


def check_finite_differences(backward, gamma, T=5, dk=3, dv=2, seed=0, with_state=True):
    """Every partial derivative against a central difference of the recurrent form."""
    rng = np.random.default_rng(seed)
    q, k, v, do, S0, dS = _inputs(rng, T, dk, dv, with_state)
    dq, dkk, dvv, dS0 = backward(q, k, v, gamma, do, S0, dS)
    S0_fd = S0 if S0 is not None else np.zeros((dk, dv))
    args = {"q": q, "k": k, "v": v, "S0": S0_fd}
    grads = {"q": dq, "k": dkk, "v": dvv, "S0": dS0}
    h = 0.5                       # the loss is affine in each entry: any step is exact
    scale = max(1.0, max(float(np.abs(g).max()) for g in grads.values()))
    for name, x in args.items():
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            a = dict(args, **{name: xp})
            b = dict(args, **{name: xm})
            fd = (_loss(a["q"], a["k"], a["v"], gamma, do, a["S0"], dS)
                  - _loss(b["q"], b["k"], b["v"], gamma, do, b["S0"], dS)) / (2 * h)
            assert abs(fd - grads[name][idx]) <= 1e-11 * scale, (name, idx, fd, grads[name][idx])


@pytest.mark.parametrize("gamma", [0.0, 0.37, 0.9, 1.0])
@pytest.mark.parametrize("with_state", [True, False])
def test_backward_matches_finite_differences(gamma, with_state):
    check_finite_differences(oracle.retention_backward, gamma, with_state=with_state)


def test_backward_finite_differences_longer():
    check_finite_differences(oracle.retention_backward, 0.8, T=9, dk=2, dv=3, seed=3)


def test_backward_gamma_zero_closed_form():
    """gamma = 0 keeps only the diagonal and the last token's state terms."""
    rng = np.random.default_rng(1)
    T, dk, dv = 6, 4, 3
    q, k, v, do, S0, dS = _inputs(rng, T, dk, dv)
    dq, dkk, dvv, dS0 = oracle.retention_backward(q, k, v, 0.0, do, S0, dS)
    for n in range(T):
        last = 1.0 if n == T - 1 else 0.0
        np.testing.assert_allclose(dq[n], np.dot(do[n], v[n]) * k[n], rtol=0, atol=1e-14)
        np.testing.assert_allclose(dkk[n], np.dot(do[n], v[n]) * q[n] + last * (dS @ v[n]),
                                   rtol=0, atol=1e-14)
        np.testing.assert_allclose(dvv[n], np.dot(q[n], k[n]) * do[n] + last * (k[n] @ dS),
                                   rtol=0, atol=1e-14)
    assert np.all(dS0 == 0.0)


def test_backward_gamma_one_cumulative_sums():
    """gamma = 1 (causal linear attention): prefix and suffix sums of outer products."""
    rng = np.random.default_rng(2)
    T, dk, dv = 8, 3, 4
    q, k, v, do, _, _ = _inputs(rng, T, dk, dv, with_state=False)
    dq, dkk, dvv, dS0 = oracle.retention_backward(q, k, v, 1.0, do)
    prefix_vk = np.cumsum(np.einsum("ti,tj->tij", v, k), axis=0)         # sum_{m<=n} v_m^T k_m
    suffix_qdo = np.cumsum(np.einsum("ti,tj->tij", q, do)[::-1], axis=0)[::-1]   # sum_{n>=m} q_n^T do_n
    np.testing.assert_allclose(dq, np.einsum("tj,tjk->tk", do, prefix_vk), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dvv, np.einsum("ti,tij->tj", k, suffix_qdo), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dkk, np.einsum("tj,tij->ti", v, suffix_qdo), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dS0, suffix_qdo[0], rtol=1e-12, atol=1e-13)


def test_backward_wrappers():
    """Multi-head and packed wrappers equal per-head, per-sequence calls."""
    rng = np.random.default_rng(4)
    H, dk, dv = 2, 3, 2
    gam = np.array([0.5, 0.95])
    lens = [5, 0, 3]
    cu = np.concatenate([[0], np.cumsum(lens)])
    Tt = int(cu[-1])
    q = rng.standard_normal((1, Tt, H, dk))
    k = rng.standard_normal((1, Tt, H, dk))
    v = rng.standard_normal((1, Tt, H, dv))
    do = rng.standard_normal((1, Tt, H, dv))
    S0 = rng.standard_normal((len(lens), H, dk, dv))
    dS = rng.standard_normal((len(lens), H, dk, dv))
    dq, dkk, dvv, dS0 = oracle.msr_backward_varlen(q, k, v, gam, do, cu, S0, dS)
    for i, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        for h in range(H):
            if b == a:
                np.testing.assert_array_equal(dS0[i, h], dS[i, h])
                continue
            r = oracle.retention_backward(q[0, a:b, h], k[0, a:b, h], v[0, a:b, h], gam[h],
                                          do[0, a:b, h], S0[i, h], dS[i, h])
            np.testing.assert_array_equal(dq[0, a:b, h], r[0])
            np.testing.assert_array_equal(dkk[0, a:b, h], r[1])
            np.testing.assert_array_equal(dvv[0, a:b, h], r[2])
            np.testing.assert_array_equal(dS0[i, h], r[3])
    b4 = oracle.msr_backward(q[:, :5], k[:, :5], v[:, :5], gam, do[:, :5], S0[:1], dS[:1])
    for x, y in zip(b4, (dq[:, :5], dkk[:, :5], dvv[:, :5], dS0[:1])):
        np.testing.assert_allclose(x, y, rtol=0, atol=0)


# ---------------------------------------------------------------------------
# Mutations: plausible mistakes planted in copies of the backward
# ---------------------------------------------------------------------------

def _backward_variant(dk_untransposed=False, in_pow_offset=1, out_reversed=False,
                      state_untransposed=False, no_state_decay=False, dv_untransposed=False):
    def f(q, k, v, gamma, d_out, state=None, d_state=None):
        q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, d_out))
        T = q.shape[0]
        D = oracle.decay_mask(gamma, T)
        A = (do @ v.T) * D
        P = (q @ k.T) * D
        dq = A @ k
        dkk = (A if dk_untransposed else A.T) @ q
        dvv = (P if dv_untransposed else P.T) @ do
        g_in = np.power(gamma, np.arange(in_pow_offset, T + in_pow_offset))
        g_out = np.power(gamma, np.arange(T) if out_reversed else np.arange(T - 1, -1, -1))
        dS0 = q.T @ (g_in[:, None] * do)
        if state is not None:
            S0 = np.asarray(state)          # square in the mutation checks (dk = dv)
            dq = dq + g_in[:, None] * (do @ (S0 if state_untransposed else S0.T))
        if d_state is not None:
            dS = np.asarray(d_state)
            dkk = dkk + g_out[:, None] * (v @ dS.T)
            dvv = dvv + g_out[:, None] * (k @ dS)
            dS0 = dS0 + (1.0 if no_state_decay else gamma ** T) * dS
        return dq, dkk, dvv, dS0
    return f


BACKWARD_MUTANTS = {
    "dK from the untransposed score matrix": _backward_variant(dk_untransposed=True),
    "dV from the untransposed score matrix": _backward_variant(dv_untransposed=True),
    "state read decays by gamma^n instead of gamma^(n+1)": _backward_variant(in_pow_offset=0),
    "final-state decays in the wrong order": _backward_variant(out_reversed=True),
    "initial-state gradient misses gamma^T": _backward_variant(no_state_decay=True),
    "state read with S0 instead of S0^T": _backward_variant(state_untransposed=True),
}


@pytest.mark.parametrize("name", list(BACKWARD_MUTANTS))
def test_finite_differences_catch_backward_mutant(name):
    mut = BACKWARD_MUTANTS[name]
    caught = False
    for gamma in (0.37, 0.9):
        try:
            check_finite_differences(mut, gamma, T=5, dk=3, dv=3)
        except AssertionError:
            caught = True
    assert caught, f"finite differences do not catch: {name}"

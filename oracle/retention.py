"""fp64 CPU oracle for Multi-Scale Retention (MSR).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, links or runs
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may call it.  It
shares no code with the CUDA library (no kernels, headers, helpers, tables or
constant generators); both sides only consume the same seeded inputs.

Everything is plain numpy in float64, written for a reader to check against
the pages by eye: no blocking, fusion or reordering beyond what each form
states.  Sources (page title, section):

* [RetNet-JA] abeam.tech summary of Sun et al. 2023, "Retentive Network: A
  Successor to Transformer for Large Language Models":
    - section 「Retentionは「内容に応じた参照」と「距離による忘却」を掛け合わせる」:
      o_n gathers the values v_m of past positions m, weighted by the content
      match Q_n K_m^T times the distance decay gamma^(n-m); future positions
      are masked.
    - section 「学習は並列、生成は状態更新」: the parallel form is Q K^T with a
      combined causal + decay mask, applied to V; the recurrent form updates a
      per-head state S_n = gamma S_(n-1) + K_n^T V_n and reads o_n = Q_n S_n;
      the state shape is fixed by the head dimensions.
    - section 「長文の学習にはチャンク再帰を使う」: chunkwise form; inside a chunk
      the interaction is parallel, past chunks arrive through the state, which
      is updated at the end of each chunk.
    - section 「多時間尺度・ゲート・正規化で表現力を補う」: each head has its own
      fixed decay rate; a Swish gate and a per-head GroupNorm follow.
* [RetNet-abs] mlnews.online abstract page for arXiv 2307.08621, summary
  bullets: retention outputs are normalised per head with GroupNorm before
  the heads are concatenated; three computation modes.
* [EulerStack] eulerwa.com EulerStack tutorial "3. RetNet 상세", sections
  "어떻게 동작하나요?" and "장점": the three modes give the same value
  (no error between training and inference forms).

Readings taken where the pages are silent (each is pinned by a test in
``tests/test_oracle.py``):

1. No 1/sqrt(d_k) scale inside retention (the formula shows none).
2. No normalisation of the decay mask or of the scores.
3. The diagonal m = n is included (gamma^0 = 1); the recurrent form updates the
   state before reading it.
4. 0^0 = 1, so gamma = 0 leaves only the diagonal term.
5. State orientation S in R^{d_k x d_v}: k_n is a 1 x d_k row, S = k^T v.
6. Chunkwise form, derived from the definition by splitting the sum over m at
   the chunk start s (row i = n - s of a chunk of length L):
     O[i] = sum_{j<=i} gamma^(i-j) (q_i . k_j) v_j + gamma^(i+1) q_i S_prev
     S    = gamma^L S_prev + sum_j gamma^(L-1-j) k_j^T v_j
   since gamma^(n-m) = gamma^(i+1) * gamma^(s-1-m) for m < s.
7. GroupNorm: groups = heads; statistics over the d_v channels of one head at
   one token; biased variance; eps added to the variance; optional affine
   weight/bias per channel (identity by default).
8. Gate: swish(x) = x * sigmoid(x), applied to the already-projected gate G
   after the GroupNorm: y = GN(o) * swish(g).
9. Variable-length batches: every sequence starts from its own initial state
   (zero by default) and is otherwise independent.

Array conventions: per-head functions take ``q, k: [T, d_k]``, ``v: [T, d_v]``
and a scalar ``gamma``; the ``msr_*`` wrappers take the token-major layout of
the library boundary, ``q, k: [B, T, H, d_k]``, ``v: [B, T, H, d_v]``,
``gamma: [H]``, and return ``o: [B, T, H, d_v]``.  States are
``[H, d_k, d_v]`` per sequence.
"""

import numpy as np

__all__ = [
    "decay_mask",
    "retention_brute",
    "retention_parallel",
    "retention_recurrent",
    "retention_chunkwise",
    "recurrent_step",
    "group_norm_heads",
    "swish",
    "norm_gate",
    "msr_parallel",
    "msr_recurrent",
    "msr_chunkwise",
    "msr_chunkwise_varlen",
    "msr_recurrent_step",
    "retention_backward",
    "msr_backward",
    "msr_backward_varlen",
    "rope",
    "softmax_features",
    "rla",
]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Per-head forms
# ---------------------------------------------------------------------------

def decay_mask(gamma, T):
    """Causal decay mask D[n, m] = gamma^(n-m) for n >= m, else 0.

    [RetNet-JA] 「学習は並列、生成は状態更新」: causal + decay mask of the parallel
    form.  Built with an integer power per entry (never gamma^n * gamma^-m).
    """
    gamma = float(gamma)
    idx = np.arange(T)
    dist = idx[:, None] - idx[None, :]          # n - m
    causal = dist >= 0
    return np.where(causal, np.power(gamma, np.where(causal, dist, 0)), 0.0)


def retention_brute(q, k, v, gamma):
    """The definition, summed term by term (tiny inputs only).

    o_n = sum_{m <= n} gamma^(n-m) (q_n . k_m) v_m
    [RetNet-JA] 「Retentionは「内容に応じた参照」と「距離による忘却」を掛け合わせる」.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, dv = q.shape[0], v.shape[1]
    gamma = float(gamma)
    o = np.zeros((T, dv), dtype=np.float64)
    for n in range(T):
        for m in range(n + 1):
            w = (gamma ** (n - m)) * float(np.dot(q[n], k[m]))
            o[n] += w * v[m]
    return o


def retention_parallel(q, k, v, gamma):
    """Parallel form O = (Q K^T * D) V.

    [RetNet-JA] 「学習は並列、生成は状態更新」 (first paragraph).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    D = decay_mask(gamma, q.shape[0])
    return ((q @ k.T) * D) @ v


def recurrent_step(q_n, k_n, v_n, gamma, S):
    """One step of the recurrent form: S <- gamma S + k_n^T v_n, then o_n = q_n S.

    [RetNet-JA] 「学習は並列、生成は状態更新」 (second paragraph).  Returns
    ``(o_n, S_new)``; ``S`` is not modified.
    """
    q_n, k_n, v_n = _f64(q_n), _f64(k_n), _f64(v_n)
    S_new = float(gamma) * _f64(S) + np.outer(k_n, v_n)
    return q_n @ S_new, S_new


def retention_recurrent(q, k, v, gamma, state=None):
    """Recurrent form over a whole sequence; returns ``(o, S_final)``."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, dk, dv = q.shape[0], q.shape[1], v.shape[1]
    S = np.zeros((dk, dv)) if state is None else _f64(state).copy()
    o = np.zeros((T, dv), dtype=np.float64)
    for n in range(T):
        o[n], S = recurrent_step(q[n], k[n], v[n], gamma, S)
    return o, S


def retention_chunkwise(q, k, v, gamma, chunk, state=None):
    """Chunkwise recurrent form; returns ``(o, S_final)``.

    [RetNet-JA] 「長文の学習にはチャンク再帰を使う」: parallel inside each chunk of
    ``chunk`` tokens, past chunks through the state, state updated at the end
    of each chunk.  Formulas: reading 6 of the module docstring.  Chunks start
    at token 0; the last one may be shorter.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, dk, dv = q.shape[0], q.shape[1], v.shape[1]
    if chunk < 1:
        raise ValueError("chunk must be >= 1")
    gamma = float(gamma)
    S = np.zeros((dk, dv)) if state is None else _f64(state).copy()
    o = np.zeros((T, dv), dtype=np.float64)
    for s in range(0, T, chunk):
        L = min(chunk, T - s)
        Qc, Kc, Vc = q[s:s + L], k[s:s + L], v[s:s + L]
        # inside the chunk: parallel form with its own decay mask
        inner = ((Qc @ Kc.T) * decay_mask(gamma, L)) @ Vc
        # past chunks: read of the carried state, decayed by gamma^(i+1)
        read_scale = np.power(gamma, np.arange(1, L + 1))          # gamma^(i+1)
        cross = read_scale[:, None] * (Qc @ S)
        o[s:s + L] = inner + cross
        # state update at the end of the chunk
        zeta = np.power(gamma, np.arange(L - 1, -1, -1))           # gamma^(L-1-j)
        S = (gamma ** L) * S + Kc.T @ (zeta[:, None] * Vc)
    return o, S


# ---------------------------------------------------------------------------
# Per-head GroupNorm and Swish gate
# ---------------------------------------------------------------------------

def group_norm_heads(o, eps=1e-5, weight=None, bias=None):
    """GroupNorm with one group per head, over the d_v channels of each token.

    ``o: [..., H, d_v]``.  [RetNet-abs] summary bullets (per-head GroupNorm
    before concatenation); [RetNet-JA] 「多時間尺度・ゲート・正規化で表現力を補う」.
    Biased variance, eps added to the variance, optional per-channel affine
    ``weight, bias: [H, d_v]``.
    """
    o = _f64(o)
    mu = o.mean(axis=-1, keepdims=True)
    var = ((o - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (o - mu) / np.sqrt(var + eps)
    if weight is not None:
        y = y * _f64(weight)
    if bias is not None:
        y = y + _f64(bias)
    return y


def swish(x):
    """swish(x) = x * sigmoid(x) = x / (1 + exp(-x))."""
    x = _f64(x)
    return x / (1.0 + np.exp(-x))


def norm_gate(o, g, eps=1e-5, weight=None, bias=None):
    """y = GroupNorm_head(o) * swish(g); ``o: [..., H, d_v]``, ``g`` same shape.

    [RetNet-JA] 「多時間尺度・ゲート・正規化で表現力を補う」 (Swish gate, GroupNorm).
    """
    g = _f64(g).reshape(np.shape(o))
    return group_norm_heads(o, eps, weight, bias) * swish(g)


# ---------------------------------------------------------------------------
# Multi-head wrappers in the boundary layout [B, T, H, d]
# ---------------------------------------------------------------------------

def _heads(q, k, v, gamma):
    q, k, v = _f64(q), _f64(k), _f64(v)
    gamma = np.asarray(gamma, dtype=np.float64).reshape(-1)
    if q.ndim != 4 or k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("expected q,k [B,T,H,dk] and v [B,T,H,dv]")
    if gamma.shape[0] != q.shape[2]:
        raise ValueError("gamma must have one entry per head")
    return q, k, v, gamma


def msr_parallel(q, k, v, gamma):
    """Parallel form for every (batch, head); multi-scale: one gamma per head."""
    q, k, v, gamma = _heads(q, k, v, gamma)
    B, T, H, _ = q.shape
    o = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            o[b, :, h] = retention_parallel(q[b, :, h], k[b, :, h], v[b, :, h], gamma[h])
    return o


def msr_recurrent(q, k, v, gamma, state=None):
    """Recurrent form for every (batch, head); returns ``(o, S [B,H,dk,dv])``."""
    q, k, v, gamma = _heads(q, k, v, gamma)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    o = np.zeros(v.shape)
    S = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            s0 = None if state is None else state[b, h]
            o[b, :, h], S[b, h] = retention_recurrent(
                q[b, :, h], k[b, :, h], v[b, :, h], gamma[h], s0)
    return o, S


def msr_chunkwise(q, k, v, gamma, chunk, state=None):
    """Chunkwise form for every (batch, head); returns ``(o, S [B,H,dk,dv])``."""
    q, k, v, gamma = _heads(q, k, v, gamma)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    o = np.zeros(v.shape)
    S = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            s0 = None if state is None else state[b, h]
            o[b, :, h], S[b, h] = retention_chunkwise(
                q[b, :, h], k[b, :, h], v[b, :, h], gamma[h], chunk, s0)
    return o, S


def msr_chunkwise_varlen(q, k, v, gamma, chunk, cu_seqlens, state=None, heads=None):
    """Packed variable-length batch: ``q,k: [1, Ttot, H, dk]``, ``v: [1, Ttot, H, dv]``.

    Sequence i occupies tokens ``cu_seqlens[i] : cu_seqlens[i+1]`` and is run
    on its own from ``state[i]`` (zero if None), chunks aligned to its first
    token (reading 9).  Returns ``(o [1,Ttot,H,dv], S [nseq,H,dk,dv])``.
    ``heads`` optionally restricts the work to a list of head indices (other
    heads' outputs are left at zero); used to sample large cases.
    """
    q, k, v, gamma = _heads(q, k, v, gamma)
    if q.shape[0] != 1:
        raise ValueError("packed layout has B = 1")
    cu = [int(x) for x in cu_seqlens]
    nseq = len(cu) - 1
    _, T, H, dk = q.shape
    dv = v.shape[3]
    o = np.zeros(v.shape)
    S = np.zeros((nseq, H, dk, dv))
    hs = range(H) if heads is None else heads
    for i in range(nseq):
        a, b = cu[i], cu[i + 1]
        for h in hs:
            s0 = None if state is None else state[i, h]
            if b > a:
                o[0, a:b, h], S[i, h] = retention_chunkwise(
                    q[0, a:b, h], k[0, a:b, h], v[0, a:b, h], gamma[h], chunk, s0)
            else:
                S[i, h] = 0.0 if s0 is None else _f64(s0)
    return o, S


def msr_recurrent_step(q, k, v, gamma, state):
    """One decode step for a batch: ``q,k: [N,H,dk]``, ``v: [N,H,dv]``,
    ``state: [N,H,dk,dv]``; returns ``(o [N,H,dv], state_new)``."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    gamma = np.asarray(gamma, dtype=np.float64).reshape(-1)
    N, H, _ = q.shape
    S = _f64(state)
    o = np.zeros(v.shape)
    S_new = np.zeros(S.shape)
    for n in range(N):
        for h in range(H):
            o[n, h], S_new[n, h] = recurrent_step(q[n, h], k[n, h], v[n, h], gamma[h], S[n, h])
    return o, S_new


# ---------------------------------------------------------------------------
# Backward: gradients of the definition (what training in the parallel form
# needs; the pages give the forward only)
# ---------------------------------------------------------------------------

def retention_backward(q, k, v, gamma, d_out, state=None, d_state=None):
    """Gradients of one head with respect to q, k, v and the initial state.

    The forward is the definition started from an initial state S0 (the
    recurrent form of [RetNet-JA] 「学習は並列、生成は状態更新」 run from S0):
        o_n = sum_{m<=n} gamma^(n-m) (q_n . k_m) v_m + gamma^(n+1) q_n S0
        S_T = gamma^T S0 + sum_m gamma^(T-1-m) k_m^T v_m
    For L = <d_out, o> + <d_state, S_T> the gradients, written with the decay
    mask D of the parallel form, are
        dQ  = ((dO V^T) * D) K         + diag(gamma^(n+1)) dO S0^T
        dK  = ((dO V^T) * D)^T Q       + diag(gamma^(T-1-m)) V dS_T^T
        dV  = ((Q K^T) * D)^T dO       + diag(gamma^(T-1-m)) K dS_T
        dS0 = Q^T diag(gamma^(n+1)) dO + gamma^T dS_T
    ``state`` / ``d_state`` of None mean zero.  Returns
    ``(dq [T,dk], dk [T,dk], dv [T,dv], d_state_in [dk,dv])``.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(d_out)
    T, dk, dv = q.shape[0], q.shape[1], v.shape[1]
    gamma = float(gamma)
    D = decay_mask(gamma, T)
    A = (do @ v.T) * D                                  # gamma^(n-m) (do_n . v_m)
    P = (q @ k.T) * D                                   # gamma^(n-m) (q_n . k_m)
    dq = A @ k
    dk_ = A.T @ q
    dv_ = P.T @ do
    g_in = np.power(gamma, np.arange(1, T + 1))         # gamma^(n+1)
    g_out = np.power(gamma, np.arange(T - 1, -1, -1))   # gamma^(T-1-m)
    dS0 = q.T @ (g_in[:, None] * do)
    if state is not None:
        dq = dq + g_in[:, None] * (do @ _f64(state).T)
    if d_state is not None:
        dS = _f64(d_state)
        dk_ = dk_ + g_out[:, None] * (v @ dS.T)
        dv_ = dv_ + g_out[:, None] * (k @ dS)
        dS0 = dS0 + (gamma ** T) * dS
    return dq, dk_, dv_, dS0


def msr_backward(q, k, v, gamma, d_out, state=None, d_state=None):
    """``retention_backward`` for every (batch, head) in the boundary layout
    ``[B, T, H, d]``; ``state``, ``d_state``: ``[B, H, dk, dv]`` or None.
    Returns ``(dq, dk, dv, d_state_in [B, H, dk, dv])``."""
    q, k, v, gamma = _heads(q, k, v, gamma)
    do = _f64(d_out)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    dq, dkk, dvv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    dS0 = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            dq[b, :, h], dkk[b, :, h], dvv[b, :, h], dS0[b, h] = retention_backward(
                q[b, :, h], k[b, :, h], v[b, :, h], gamma[h], do[b, :, h],
                None if state is None else state[b, h],
                None if d_state is None else d_state[b, h])
    return dq, dkk, dvv, dS0


def msr_backward_varlen(q, k, v, gamma, d_out, cu_seqlens, state=None, d_state=None,
                        heads=None):
    """Packed variable-length batch (``B = 1``, sequences at ``cu_seqlens``):
    every sequence is differentiated on its own (reading 9).  ``state``,
    ``d_state``: ``[nseq, H, dk, dv]`` or None; an empty sequence passes
    ``d_state`` straight to its ``d_state_in``.  ``heads`` optionally restricts
    the work to a list of heads."""
    q, k, v, gamma = _heads(q, k, v, gamma)
    do = _f64(d_out)
    cu = [int(x) for x in cu_seqlens]
    nseq = len(cu) - 1
    _, T, H, dk = q.shape
    dv = v.shape[3]
    dq, dkk, dvv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    dS0 = np.zeros((nseq, H, dk, dv))
    hs = range(H) if heads is None else heads
    for i in range(nseq):
        a, b = cu[i], cu[i + 1]
        for h in hs:
            s0 = None if state is None else state[i, h]
            dS = None if d_state is None else d_state[i, h]
            if b > a:
                dq[0, a:b, h], dkk[0, a:b, h], dvv[0, a:b, h], dS0[i, h] = retention_backward(
                    q[0, a:b, h], k[0, a:b, h], v[0, a:b, h], gamma[h], do[0, a:b, h], s0, dS)
            else:
                dS0[i, h] = 0.0 if dS is None else _f64(dS)
    return dq, dkk, dvv, dS0


# ---------------------------------------------------------------------------
# Rotary position encoding of q and k
# ---------------------------------------------------------------------------

def rope(x, base=10000.0, cu_seqlens=None):
    """Rotary position encoding of ``x: [B, T, H, d]`` (d even), in float64.

    [RetNet-JA] 「Retentionは「内容に応じた参照」と「距離による忘却」を掛け合わせる」:
    Q and K receive a position rotation after the projections; [EulerStack]
    "장점": RoPE-compatible.  The pages give no formula; the reading taken is
    the standard rotary form: the pair (x[2i], x[2i+1]) of a token at position
    p (its index within its own sequence) is rotated by the angle p * theta_i,
    theta_i = base^(-2i/d):
        x'[2i]   = x[2i] cos(p theta_i) - x[2i+1] sin(p theta_i)
        x'[2i+1] = x[2i] sin(p theta_i) + x[2i+1] cos(p theta_i)
    Packed sequences (``B = 1`` and ``cu_seqlens``) count positions from each
    sequence's first token.
    """
    x = _f64(x)
    B, T, H, d = x.shape
    if d % 2:
        raise ValueError("rope needs an even head dimension")
    pos = np.zeros((B, T))
    if cu_seqlens is None:
        pos[:] = np.arange(T)[None, :]
    else:
        cu = [int(c) for c in cu_seqlens]
        for a, b in zip(cu[:-1], cu[1:]):
            pos[0, a:b] = np.arange(b - a)
    theta = np.power(float(base), -np.arange(0, d, 2) / d)          # [d/2]
    ang = pos[:, :, None, None] * theta[None, None, None, :]         # [B, T, 1, d/2]
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# ---------------------------------------------------------------------------
# Residual linear attention (RLA): the linear-attention state read w tokens late
# ---------------------------------------------------------------------------

def softmax_features(x):
    """Feature map phi(x) = softmax over the last axis (the head dimension).

    The RAttention page (section "Residual Linear Attention (RLA) 수식") names a
    feature map phi and calls a softmax-based one the best choice, without a
    formula; the reading taken is the row softmax of each (token, head) vector.
    """
    x = _f64(x)
    e = np.exp(x - x.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def rla(q, k, v, window, cu_seqlens=None):
    """Residual linear attention of ``q, k: [B,T,H,dk]``, ``v: [B,T,H,dv]``.

    RAttention page, section "Residual Linear Attention (RLA) 수식": a state
    without decay, S_t = S_(t-1) + phi(k_t)^T v_t, read w tokens late,
    o_t = phi(q_t) S_(t-w-1), with S of a position before the sequence = 0
    (reading: the window w >= 0 counts the tokens the read skips, so o_t sees
    tokens m <= t - w - 1).  Run per (sequence, head) as the recurrence written
    on the page, with phi evaluated in float64.  Returns ``o [B,T,H,dv]``.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    fq, fk = softmax_features(q), softmax_features(k)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    o = np.zeros((B, T, H, dv))
    segs = ([(b, 0, T) for b in range(B)] if cu_seqlens is None
            else [(0, int(a), int(e)) for a, e in zip(cu_seqlens[:-1], cu_seqlens[1:])])
    for b, a, e in segs:
        for h in range(H):
            # S_(t-w-1), built by the same recurrence running w+1 tokens behind t
            S = np.zeros((dk, dv))
            for t in range(a, e):
                m = t - window - 1
                if m >= a:
                    S = S + np.outer(fk[b, m, h], v[b, m, h])
                    o[b, t, h] = fq[b, t, h] @ S
    return o

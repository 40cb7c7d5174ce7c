"""Parity at the workloads' full sizes, in the launch configuration bench.py
times, checked against the fp64 oracle on sampled (sequence, head) pairs.

Inputs follow the shared recipe of linear_recurrent_sequence_retention_b200.
workloads (q, k, v ~ N(0,1)/sqrt(d_k), g ~ N(0,1), seeded); the large ones are
drawn on the device with a seeded torch CUDA generator and the sampled
slices are copied to the host for the oracle.  Tolerance (bf16 inputs,
f32 accumulation): relative L2 <= 1e-2 and max-abs <= 3e-2 * RMS per sampled
head; outputs stored as bf16 add their own rounding (tests/_util.py).
"""

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_sequence_retention_b200 import ops, workloads as W
from tests._util import assert_close

pytestmark = pytest.mark.gpu

f64 = W.to_f64


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    torch.cuda.empty_cache()


def test_msr_b4_h8_t2048_gated_full_size():
    wl = W.WORKLOADS["msr_b4_h8_t2048_dk128_dv256_c128"]
    q, k, v, g = W.make_qkvg(wl.B, wl.T, wl.H, wl.dk, wl.dv, "bf16", seed=0)
    gam = W.head_gammas(wl.H)
    y = ops.chunkwise_fwd(q.cuda(), k.cuda(), v.cuda(), gam, wl.chunk, g=g.cuda())
    ops.check_device_error()
    y = f64(y)
    assert np.isfinite(y).all()
    gg = f64(g).reshape(wl.B, wl.T, wl.H, wl.dv)
    for b, h in [(0, 0), (1, 3), (2, 5), (3, 7)]:
        o, _ = oracle.retention_chunkwise(f64(q[b, :, h]), f64(k[b, :, h]), f64(v[b, :, h]),
                                          gam[h], wl.chunk)
        ref = oracle.norm_gate(o[:, None, :], gg[b, :, h][:, None, :])[:, 0]
        assert_close(y[b, :, h], ref, "bf16", None, f"y b={b} h={h}", stored_bf16=True)


def test_msr_6p7b_t8192_gated_state_full_size():
    wl = W.WORKLOADS["msr_6p7b_b2_h16_t8192_dk256_dv512_c512"]
    q, k, v, g = W.make_qkvg(wl.B, wl.T, wl.H, wl.dk, wl.dv, "bf16", seed=0, device="cuda")
    gam = W.head_gammas(wl.H)
    y, S = ops.chunkwise_fwd(q, k, v, gam, wl.chunk, g=g, return_state=True)
    ops.check_device_error()
    assert bool(torch.isfinite(y).all()) and bool(torch.isfinite(S).all())
    for b, h in [(0, 0), (1, 15), (0, 8), (1, 4)]:
        qb, kb, vb = f64(q[b, :, h]), f64(k[b, :, h]), f64(v[b, :, h])
        o, S_ref = oracle.retention_chunkwise(qb, kb, vb, gam[h], wl.chunk)
        gb = f64(g[b].reshape(wl.T, wl.H, wl.dv)[:, h])
        ref = oracle.norm_gate(o[:, None, :], gb[:, None, :])[:, 0]
        assert_close(f64(y[b, :, h]), ref, "bf16", None, f"y b={b} h={h}", stored_bf16=True)
        assert_close(f64(S[b, h]), S_ref, "bf16", None, f"state b={b} h={h}")


def test_msr_6p7b_t8192_f32_out_plain_bound():
    """The 6.7B-shaped workload at full size (T = 8192) with the output written
    as float32 by the same kernels: the plain bound (rel-L2 <= 1e-2, max-abs <=
    3e-2 * RMS) with no allowance for a bf16 store, on sampled (sequence, head)
    pairs that include the fastest- and the slowest-decaying head."""
    wl = W.WORKLOADS["msr_6p7b_b2_h16_t8192_dk256_dv512_c512"]
    q, k, v, g = W.make_qkvg(wl.B, wl.T, wl.H, wl.dk, wl.dv, "bf16", seed=0, device="cuda")
    gam = W.head_gammas(wl.H)
    y, S = ops.chunkwise_fwd(q, k, v, gam, wl.chunk, g=g, return_state=True,
                             out_dtype=torch.float32)
    ops.check_device_error()
    assert y.dtype == torch.float32
    assert bool(torch.isfinite(y).all()) and bool(torch.isfinite(S).all())
    for b, h in [(0, 0), (1, 15), (1, 1), (0, 11)]:
        qb, kb, vb = f64(q[b, :, h]), f64(k[b, :, h]), f64(v[b, :, h])
        o, S_ref = oracle.retention_chunkwise(qb, kb, vb, gam[h], wl.chunk)
        gb = f64(g[b].reshape(wl.T, wl.H, wl.dv)[:, h])
        ref = oracle.norm_gate(o[:, None, :], gb[:, None, :])[:, 0]
        assert_close(f64(y[b, :, h]), ref, "bf16", None, f"y f32 b={b} h={h}")
        assert_close(f64(S[b, h]), S_ref, "bf16", None, f"state b={b} h={h}")


def test_decode_after_full_prefill():
    """128 sequences x 16 heads: state-only chunkwise prefill of 8192 tokens (in
    groups of 16 sequences, as bench.py does), then decode steps on the whole
    batch; sampled sequences checked against the oracle's prefill + steps."""
    wl = W.WORKLOADS["decode_6p7b_n128_h16_dk256_dv512"]
    N, H, dk, dv = wl.B, wl.H, wl.dk, wl.dv
    gam = W.head_gammas(H)
    S = torch.empty(N, H, dk, dv, device="cuda")
    grp = 16
    sampled = {0: None, 77: None}
    ws = None
    for n0 in range(0, N, grp):
        _, kk, vv, _ = W.make_qkvg(grp, wl.T, H, dk, dv, "bf16", seed=500 + n0, gate=False,
                                   device="cuda")
        if ws is None:
            ws = ops.alloc_workspace(ops.chunkwise_workspace_size(torch.bfloat16, wl.chunk, grp,
                                                                  wl.T, H, dk, dv), "cuda")
        ops.chunkwise_states(kk, vv, gam, wl.chunk, state_out=S[n0:n0 + grp], workspace=ws)
        for n in sampled:
            if n0 <= n < n0 + grp:
                sampled[n] = (f64(kk[n - n0]), f64(vv[n - n0]))
        del kk, vv
    ops.check_device_error()
    steps = 8
    o_gpu, steps_in = [], []
    for t in range(steps):
        qs, ks, vs = W.make_step_inputs(N, H, dk, dv, "bf16", seed=900 + t, device="cuda")
        o_gpu.append(f64(ops.recurrent_step(qs, ks, vs, gam, S)))
        steps_in.append((f64(qs), f64(ks), f64(vs)))
    ops.check_device_error()
    S_gpu = f64(S)
    for n, (kn, vn) in sampled.items():
        for h in (0, 9, 15):
            _, Sr = oracle.retention_chunkwise(np.zeros((wl.T, dk)), kn[:, h], vn[:, h],
                                               gam[h], wl.chunk)
            for t in range(steps):
                qs, ks, vs = steps_in[t]
                o_ref, Sr = oracle.recurrent_step(qs[n, h], ks[n, h], vs[n, h], gam[h], Sr)
                assert_close(o_gpu[t][n, h], o_ref, "bf16", None, f"o n={n} h={h} t={t}")
            assert_close(S_gpu[n, h], Sr, "bf16", None, f"state n={n} h={h}")


def test_varlen_64seq_full_size():
    wl = W.WORKLOADS["varlen_64seq_h8_d128_c64"]
    nseq, lo, hi = wl.varlen
    lens = W.varlen_lengths(nseq, lo, hi, seed=0)
    cu = W.cu_seqlens_of(lens)
    Tt = int(cu[-1])
    q, k, v, _ = W.make_qkvg(1, Tt, wl.H, wl.dk, wl.dv, "bf16", seed=0, gate=False, device="cuda")
    gam = W.head_gammas(wl.H)
    o, S = ops.chunkwise_fwd(q, k, v, gam, wl.chunk, cu_seqlens=torch.from_numpy(cu).cuda(),
                             return_state=True)
    ops.check_device_error()
    assert bool(torch.isfinite(o).all())
    longest = int(np.argmax(lens))
    for i, h in [(0, 0), (longest, 7), (nseq - 1, 3)]:
        a, b = int(cu[i]), int(cu[i + 1])
        o_ref, S_ref = oracle.retention_chunkwise(f64(q[0, a:b, h]), f64(k[0, a:b, h]),
                                                  f64(v[0, a:b, h]), gam[h], wl.chunk)
        assert_close(f64(o[0, a:b, h]), o_ref, "bf16", None, f"o seq={i} h={h}", stored_bf16=True)
        assert_close(f64(S[i, h]), S_ref, "bf16", None, f"state seq={i} h={h}")

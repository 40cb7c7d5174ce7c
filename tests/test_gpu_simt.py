"""GPU parity of the CUDA-core kernels against the fp64 oracle, through the C ABI:
float32 parallel / recurrent / chunkwise forms (tolerance: relative L2 <= 1e-5),
the decode step, the standalone GroupNorm + gate, and the device error word."""

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_sequence_retention_b200 import ops, workloads as W
from tests._util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()
    yield
    ops.check_device_error()


def _f64(t):
    return W.to_f64(t)


def test_tiny_fp32_parallel_recurrent_chunkwise():
    """The tiny float32 workload: all three forms against the oracle."""
    wl = W.WORKLOADS["tiny_fp32_b1_h2_t64_d16_c16"]
    q, k, v, _ = W.make_qkvg(wl.B, wl.T, wl.H, wl.dk, wl.dv, "f32", gate=False)
    gam = W.head_gammas(wl.H)
    ref_o, ref_S = oracle.msr_chunkwise(_f64(q), _f64(k), _f64(v), gam, wl.chunk)
    assert_close(ref_o, oracle.msr_parallel(_f64(q), _f64(k), _f64(v), gam), "f32", 2, "oracle")
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o_par = ops.parallel_fwd(qd, kd, vd, gam)
    assert_close(_f64(o_par), ref_o, "f32", 2, "parallel")
    o_chk, S_chk = ops.chunkwise_fwd(qd, kd, vd, gam, wl.chunk, return_state=True)
    assert_close(_f64(o_chk), ref_o, "f32", 2, "chunkwise")
    assert_close(_f64(S_chk), ref_S, "f32", 1, "chunkwise state")
    S = torch.zeros(wl.B, wl.H, wl.dk, wl.dv, device="cuda")
    outs = []
    for t in range(wl.T):
        outs.append(ops.recurrent_step(qd[:, t].contiguous(), kd[:, t].contiguous(),
                                       vd[:, t].contiguous(), gam, S))
    o_rec = torch.stack(outs, dim=1)
    assert_close(_f64(o_rec), ref_o, "f32", 2, "recurrent")
    assert_close(_f64(S), ref_S, "f32", 1, "recurrent state")


@pytest.mark.parametrize("B,T,chunk,dk,dv", [
    (2, 37, 1, 8, 8),       # chunk of one token
    (1, 37, 3, 16, 24),     # ragged tail
    (2, 50, 16, 24, 40),    # dk != dv, several chunks
    (1, 5, 16, 16, 16),     # T < chunk
    (1, 1, 4, 8, 8),        # single token
    (3, 70, 64, 32, 32),    # chunk > tail
    (1, 300, 128, 64, 256), # wide values, several tiles
])
def test_fp32_chunkwise_shapes(B, T, chunk, dk, dv):
    H = 3
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "f32", seed=B * 1000 + T, gate=False)
    gam = np.array([0.0, 0.9, 1.0])     # includes the gamma = 0 and gamma = 1 extremes
    s0 = W.make_state(B, H, dk, dv, seed=3, scale=0.1)
    ref_o, ref_S = oracle.msr_chunkwise(_f64(q), _f64(k), _f64(v), gam, chunk, _f64(s0))
    o, S = ops.chunkwise_fwd(q.cuda(), k.cuda(), v.cuda(), gam, chunk, state_in=s0.cuda(),
                             return_state=True)
    assert_close(_f64(o), ref_o, "f32", 2, "o")
    assert_close(_f64(S), ref_S, "f32", 1, "state")
    o2 = ops.parallel_fwd(q.cuda(), k.cuda(), v.cuda(), gam)
    ref_p = oracle.msr_parallel(_f64(q), _f64(k), _f64(v), gam)
    assert_close(_f64(o2), ref_p, "f32", 2, "parallel")


def test_fp32_chunk_length_invariance():
    """The result does not depend on the chunk length (the three forms agree)."""
    B, T, H, dk, dv = 1, 96, 2, 16, 16
    q, k, v, _ = W.make_qkvg(B, T, H, dk, dv, "f32", seed=5, gate=False)
    gam = W.head_gammas(H)
    ref = oracle.msr_parallel(_f64(q), _f64(k), _f64(v), gam)
    for chunk in (1, 7, 16, 32, 96, 200):
        o = ops.chunkwise_fwd(q.cuda(), k.cuda(), v.cuda(), gam, chunk)
        assert_close(_f64(o), ref, "f32", 2, f"chunk={chunk}")


def test_fp32_varlen_packed():
    lens = [5, 0, 17, 1, 40, 23]
    cu = W.cu_seqlens_of(lens)
    H, dk, dv, chunk = 2, 16, 8, 8
    Tt = int(cu[-1])
    q, k, v, _ = W.make_qkvg(1, Tt, H, dk, dv, "f32", seed=9, gate=False)
    s0 = W.make_state(len(lens), H, dk, dv, seed=4, scale=0.2)
    gam = np.array([0.8, 0.97])
    ref_o, ref_S = oracle.msr_chunkwise_varlen(_f64(q), _f64(k), _f64(v), gam, chunk, cu, _f64(s0))
    o, S = ops.chunkwise_fwd(q.cuda(), k.cuda(), v.cuda(), gam, chunk,
                             cu_seqlens=torch.from_numpy(cu).cuda(), state_in=s0.cuda(),
                             return_state=True)
    assert_close(_f64(o), ref_o, "f32", 2, "o")
    assert_close(_f64(S), ref_S, "f32", 1, "state")
    np.testing.assert_array_equal(_f64(S)[1], _f64(s0)[1])   # empty sequence: state passes through
    ops.check_device_error()


def test_fp32_chunkwise_gated():
    B, T, H, dk, dv, chunk = 2, 45, 3, 16, 32, 16
    q, k, v, g = W.make_qkvg(B, T, H, dk, dv, "f32", seed=21)
    gam = W.head_gammas(H)
    w = torch.randn(H * dv, generator=torch.Generator().manual_seed(1))
    b = torch.randn(H * dv, generator=torch.Generator().manual_seed(2))
    o_ref, _ = oracle.msr_chunkwise(_f64(q), _f64(k), _f64(v), gam, chunk)
    y_ref = oracle.norm_gate(o_ref, _f64(g).reshape(B, T, H, dv), 1e-5,
                             _f64(w).reshape(H, dv), _f64(b).reshape(H, dv))
    y = ops.chunkwise_fwd(q.cuda(), k.cuda(), v.cuda(), gam, chunk, g=g.cuda(),
                          gn_weight=w.cuda(), gn_bias=b.cuda())
    assert_close(_f64(y), y_ref, "f32", 2, "y")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,H,dk,dv", [(4, 3, 64, 96), (2, 2, 256, 512), (3, 1, 17, 10)])
def test_decode_step(dtype, N, H, dk, dv):
    """Decode arithmetic is float32 even for bf16 inputs (the oracle consumes the
    same bf16-rounded values), so the float32 tolerance applies."""
    gam = np.linspace(0.5, 1.0, H)
    S = W.make_state(N, H, dk, dv, seed=N + dk, scale=0.3)
    S_ref = _f64(S)
    Sd = S.cuda()
    for step in range(3):
        q, k, v = W.make_step_inputs(N, H, dk, dv, dtype, seed=step)
        o = ops.recurrent_step(q.cuda(), k.cuda(), v.cuda(), gam, Sd)
        o_ref, S_ref = oracle.msr_recurrent_step(_f64(q), _f64(k), _f64(v), gam, S_ref)
        assert_close(_f64(o), o_ref, "f32", 1, f"o step {step}")
        assert_close(_f64(Sd), S_ref, "f32", 1, f"state step {step}")


@pytest.mark.parametrize("o_dt,y_dt,dv", [("f32", "f32", 64), ("bf16", "bf16", 512),
                                          ("f32", "bf16", 96), ("bf16", "f32", 33)])
def test_norm_gate(o_dt, y_dt, dv):
    ntok, H = 37, 3
    gen = torch.Generator().manual_seed(dv)
    o = (torch.randn(ntok, H, dv, generator=gen) * 2 + 0.5).to(W.torch_dtype(o_dt))
    g = torch.randn(ntok, H * dv, generator=gen).to(W.torch_dtype(o_dt))
    w = torch.randn(H * dv, generator=gen)
    b = torch.randn(H * dv, generator=gen)
    ref = oracle.norm_gate(_f64(o), _f64(g).reshape(ntok, H, dv), 1e-5,
                           _f64(w).reshape(H, dv), _f64(b).reshape(H, dv))
    y = ops.norm_gate(o.cuda(), g.cuda(), w.cuda(), b.cuda(), out_dtype=W.torch_dtype(y_dt))
    kind = "f32" if y_dt == "f32" else "bf16"   # inputs are exact; only a bf16 store rounds
    assert_close(_f64(y), ref, kind, 1, "y", stored_bf16=(y_dt == "bf16"))
    y0 = ops.norm_gate(o.cuda(), torch.zeros_like(g).cuda())
    assert float(y0.abs().max()) == 0.0


def test_malformed_cu_seqlens_reported_not_faulted():
    """Non-monotone offsets: kernels clamp every access, the error word says so."""
    H, dk, dv = 2, 8, 8
    q, k, v, _ = W.make_qkvg(1, 20, H, dk, dv, "f32", seed=1, gate=False)
    cu = torch.tensor([0, 15, 5, 30], dtype=torch.int32).cuda()
    o = torch.zeros(1, 20, H, dv, device="cuda")     # rows outside every range stay untouched
    ops.chunkwise_fwd(q.cuda(), k.cuda(), v.cuda(), [0.9, 0.9], 8, cu_seqlens=cu, out=o)
    with pytest.raises(ops.RetentionError) as ei:
        ops.check_device_error()
    assert ei.value.status == ops.RET_ERR_DEVICE_DATA
    assert torch.isfinite(o).all()
    ops.check_device_error()            # the word was cleared by the previous read
